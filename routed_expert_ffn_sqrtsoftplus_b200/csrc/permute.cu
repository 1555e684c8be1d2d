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

constexpr int kMaxGroups = 1024;

__global__ void __launch_bounds__(256)
    perm_count_kernel(const int32_t* __restrict__ idx, int nslots, int E, int32_t* __restrict__ chunk_cnt,
                      int* status) {
  __shared__ int hist[kMaxGroups];
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const int base = blockIdx.x * kPermChunk;
  const int end = min(nslots, base + kPermChunk);
  for (int s = base + threadIdx.x; s < end; s += blockDim.x) {
    const int e = idx[s];
    if (e >= 0 && e < E)
      atomicAdd(&hist[e], 1);
    else
      report_status(status, kStatusDevice);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) chunk_cnt[static_cast<size_t>(blockIdx.x) * E + e] = hist[e];
}

__global__ void __launch_bounds__(1024) perm_scan_kernel(ScanArgs a) {
  __shared__ int cnt_s[kMaxGroups];
  __shared__ int off_s[kMaxGroups + 1];
  __shared__ int tgu_s[kMaxGroups + 1];
  __shared__ int tdn_s[kMaxGroups + 1];
  __shared__ int ngu_s[kMaxGroups + 1];
  __shared__ int ndn_s[kMaxGroups + 1];
  const int G = a.E + a.S;
  // 1. per-expert totals and per-chunk running counts (relative bases)
  for (int g = threadIdx.x; g < G; g += blockDim.x) {
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
  __syncthreads();
  // 2. exclusive scans over groups (serial: G <= 1024)
  if (threadIdx.x == 0) {
    int o = 0, tg = 0, td = 0, ng = 0, nd = 0;
    // tile lists visit the shared experts first, then the routed experts
    for (int r = 0; r < G; ++r) {
      const int g = r < a.S ? a.E + r : r - a.S;
      const int n = cnt_s[g];
      const bool sh = g >= a.E;
      const int bgu = sh ? a.bn_gu_s : a.bn_gu_r, bdn = sh ? a.bn_dn_s : a.bn_dn_r;
      const int ntg = (n + bgu - 1) / bgu, ntd = (n + bdn - 1) / bdn;
      tgu_s[g] = tg;
      tdn_s[g] = td;
      tg += a.m_tiles_gu * ntg;
      td += a.m_tiles_dn * ntd;
      if (r == a.S - 1) {
        a.ntiles[2] = tg;
        a.ntiles[3] = td;
      }
      if (!sh) {
        ngu_s[g] = ng;
        ndn_s[g] = nd;
        ng += ntg;
        nd += ntd;
      }
    }
    if (a.S == 0) {
      a.ntiles[2] = 0;
      a.ntiles[3] = 0;
    }
    ngu_s[a.E] = ng;
    ndn_s[a.E] = nd;
    for (int g = 0; g < G; ++g) {
      off_s[g] = o;
      o += cnt_s[g];
    }
    off_s[G] = o;
    a.ntiles[0] = tg;
    a.ntiles[1] = td;
  }
  __syncthreads();
  // 3. outputs
  for (int g = threadIdx.x; g <= G; g += blockDim.x) {
    a.off[g] = off_s[g];
    if (g < G) a.cnt[g] = cnt_s[g];
  }
  if (a.ntile_base_gu != nullptr)
    for (int g = threadIdx.x; g <= a.E; g += blockDim.x) {
      a.ntile_base_gu[g] = ngu_s[g];
      a.ntile_base_dn[g] = ndn_s[g];
    }
  for (int g = threadIdx.x; g < a.E; g += blockDim.x)
    for (int c = 0; c < a.nchunks; ++c) a.chunk_cnt[static_cast<size_t>(c) * a.E + g] += off_s[g];
  for (int g = threadIdx.x; g < G; g += blockDim.x) {
    const int n = cnt_s[g];
    const bool shared = g >= a.E;
    const bool mx = a.mx && !shared;
    // gate/up tiles: m-major, token tiles of one weight tile adjacent
    int bn = shared ? a.bn_gu_s : a.bn_gu_r;
    int ntn = (n + bn - 1) / bn;
    int pos = tgu_s[g];
    for (int mt = 0; mt < a.m_tiles_gu; ++mt)
      for (int nt = 0; nt < ntn; ++nt) {
        const int r0 = nt * bn;
        const int y = mx ? ngu_s[g] + nt : (shared ? r0 : off_s[g] + r0);
        a.tiles_gu[pos++] = make_int4(g | (mt << 16), y, off_s[g] + r0, min(bn, n - r0));
      }
    bn = shared ? a.bn_dn_s : a.bn_dn_r;
    ntn = (n + bn - 1) / bn;
    pos = tdn_s[g];
    for (int mt = 0; mt < a.m_tiles_dn; ++mt)
      for (int nt = 0; nt < ntn; ++nt) {
        const int r0 = nt * bn;
        const int y = mx ? ndn_s[g] + nt : off_s[g] + r0;
        a.tiles_dn[pos++] = make_int4(g | (mt << 16), y, off_s[g] + r0, min(bn, n - r0));
      }
  }
}

// One warp per chunk walks its slots in order, 32 at a time; peers with the
// same expert get consecutive positions in lane order.
__global__ void __launch_bounds__(32)
    perm_scatter_kernel(const int32_t* __restrict__ idx, int nslots, int E, const int32_t* __restrict__ chunk_base,
                        int32_t* __restrict__ perm, int32_t* __restrict__ inv) {
  __shared__ int ctr[kMaxGroups];
  const int lane = threadIdx.x;
  for (int e = lane; e < E; e += 32) ctr[e] = chunk_base[static_cast<size_t>(blockIdx.x) * E + e];
  __syncwarp();
  const int base = blockIdx.x * kPermChunk;
  const int end = min(nslots, base + kPermChunk);
  for (int b = base; b < end; b += 32) {
    const int s = b + lane;
    const int e = s < end ? idx[s] : -1;
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
    gather_rows_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ perm, int nrows, int k, int hv,
                       uint4* __restrict__ xp) {
  const int row = blockIdx.x * 8 + threadIdx.x / 32;
  if (row >= nrows) return;
  const int t = perm[row] / k;
  const uint4* src = x + static_cast<size_t>(t) * hv;
  uint4* dst = xp + static_cast<size_t>(row) * hv;
  for (int c = threadIdx.x % 32; c < hv; c += 32) dst[c] = __ldg(src + c);
}

// MXFP8 quantisation of the routed token rows (OCP MX v1.0 rule, E4M3 with
// round-to-nearest-even and saturation): one warp per row, one 32-value block
// per lane per step. The E8M0 codes go straight into the scale-factor atoms of
// the gate/up token tile that holds the row.
__global__ void __launch_bounds__(256)
    quant_gather_mx_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ perm,
                           const int32_t* __restrict__ idx, const int32_t* __restrict__ off,
                           const int32_t* __restrict__ ntile_base, int nrows, int k, int H, int bn,
                           uint4* __restrict__ xq, uint8_t* __restrict__ sfb) {
  const int row = blockIdx.x * 8 + threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  if (row >= nrows) return;
  const int slot = perm[row];
  const int t = slot / k;
  const int g = idx[slot];
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
                                   const int32_t* ntile_base_gu, int nrows, int k, int H, int bn_gu, uint8_t* xq,
                                   uint8_t* sfb, cudaStream_t s) {
  if (nrows == 0) return cudaSuccess;
  quant_gather_mx_kernel<<<(nrows + 7) / 8, 256, 0, s>>>(static_cast<const uint4*>(x), perm, idx, off,
                                                          ntile_base_gu, nrows, k, H, bn_gu,
                                                          reinterpret_cast<uint4*>(xq), sfb);
  return cudaGetLastError();
}

cudaError_t launch_perm_count(const int32_t* idx, int nslots, int E, int32_t* chunk_cnt, int* status,
                              cudaStream_t s) {
  if (E > kMaxGroups) return cudaErrorInvalidValue;
  const int nchunks = (nslots + kPermChunk - 1) / kPermChunk;
  perm_count_kernel<<<nchunks, 256, 0, s>>>(idx, nslots, E, chunk_cnt, status);
  return cudaGetLastError();
}

cudaError_t launch_perm_scan(const ScanArgs& a, cudaStream_t s) {
  if (a.E + a.S > kMaxGroups) return cudaErrorInvalidValue;
  perm_scan_kernel<<<1, 1024, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_perm_scatter(const int32_t* idx, int nslots, int E, const int32_t* chunk_base, int32_t* perm,
                                int32_t* inv, cudaStream_t s) {
  const int nchunks = (nslots + kPermChunk - 1) / kPermChunk;
  perm_scatter_kernel<<<nchunks, 32, 0, s>>>(idx, nslots, E, chunk_base, perm, inv);
  return cudaGetLastError();
}

cudaError_t launch_gather_rows(const void* x, const int32_t* perm, int nrows, int k, int H, void* xp,
                               cudaStream_t s) {
  if (nrows == 0) return cudaSuccess;
  gather_rows_kernel<<<(nrows + 7) / 8, 256, 0, s>>>(static_cast<const uint4*>(x), perm, nrows, k, H / 8,
                                                     static_cast<uint4*>(xp));
  return cudaGetLastError();
}

}  // namespace moe
