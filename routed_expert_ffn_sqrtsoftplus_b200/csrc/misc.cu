// Weighted combine with the shared experts, weight repacking, the MXFP4 weight
// quantiser utility, and the bounded-wait self test.
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

// y[t] = sum_shared O[T*k + j*T + t] + sum_j w[t, j] * O[inv[t*k + j]]
// (shared experts have weight 1; the routed sum runs in slot order j = 0..k-1,
// accumulated in fp32 and rounded once to BF16). Only slots whose expert lies in
// this instance's window [e_begin, e_begin + e_count) count (all of them for a
// whole layer); with y_f32 the sum is written in fp32 (an expert-parallel
// partial output, summed over the instances afterwards).
constexpr int kCombineMaxK = 32;   // top_k <= 32
constexpr int kCombineBatch = 8;   // O rows loaded before their products are summed

__global__ void __launch_bounds__(128)
    combine_kernel(const float4* __restrict__ O, const int32_t* __restrict__ inv, const int32_t* __restrict__ idx,
                   int e_begin, int e_count, const float* __restrict__ w, int T, int H4, int k, int S,
                   void* __restrict__ y, int y_f32, const float4* __restrict__ sh_parts, int n_parts) {
  // the token's slots, read once per block: O row (-1: another instance's expert, or
  // a row index outside O, which only corrupted memory could give) and weight
  __shared__ int row_s[kCombineMaxK];
  __shared__ float w_s[kCombineMaxK];
  const int t = blockIdx.x;
  const size_t routed_rows = static_cast<size_t>(T) * k;
  if (static_cast<int>(threadIdx.x) < k) {
    const size_t i = static_cast<size_t>(t) * k + threadIdx.x;
    const int e = __ldg(idx + i) - e_begin;
    const int row = __ldg(inv + i);
    const bool use = e >= 0 && e < e_count && row >= 0 && static_cast<size_t>(row) < routed_rows;
    row_s[threadIdx.x] = use ? row : -1;
    w_s[threadIdx.x] = __ldg(w + i);
  }
  __syncthreads();
  const int c = blockIdx.y * blockDim.x + threadIdx.x;
  if (c >= H4) return;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int j = 0; j < S; ++j) {
    if (sh_parts == nullptr) {
      const float4 v = __ldg(O + (routed_rows + static_cast<size_t>(j) * T + t) * H4 + c);
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    } else {
      // split-K slices of shared expert j, summed in slice order
      float4 sj = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int p = 0; p < n_parts; ++p) {
        const float4 v = __ldg(sh_parts + ((static_cast<size_t>(j) * n_parts + p) * T + t) * H4 + c);
        sj.x += v.x;
        sj.y += v.y;
        sj.z += v.z;
        sj.w += v.w;
      }
      acc.x += sj.x;
      acc.y += sj.y;
      acc.z += sj.z;
      acc.w += sj.w;
    }
  }
  // routed slots in slot order; a batch of rows is in flight at once
  for (int j0 = 0; j0 < k; j0 += kCombineBatch) {
    float4 v[kCombineBatch];
#pragma unroll
    for (int u = 0; u < kCombineBatch; ++u) {
      const int row = j0 + u < k ? row_s[j0 + u] : -1;
      v[u] = row >= 0 ? __ldg(O + static_cast<size_t>(row) * H4 + c) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < kCombineBatch; ++u) {
      if (j0 + u < k && row_s[j0 + u] >= 0) {
        const float wj = w_s[j0 + u];
        acc.x = fmaf(wj, v[u].x, acc.x);
        acc.y = fmaf(wj, v[u].y, acc.y);
        acc.z = fmaf(wj, v[u].z, acc.z);
        acc.w = fmaf(wj, v[u].w, acc.w);
      }
    }
  }
  if (y_f32) {
    static_cast<float4*>(y)[static_cast<size_t>(t) * H4 + c] = acc;
    return;
  }
  __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
  __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
  uint2 out;
  out.x = *reinterpret_cast<uint32_t*>(&lo);
  out.y = *reinterpret_cast<uint32_t*>(&hi);
  static_cast<uint2*>(y)[static_cast<size_t>(t) * H4 + c] = out;
}

// h[t, i] = silu(min(G, L)) * clamp(U, -L, L) with G, U the sums of the split-K
// slices parts[p][t][i] and parts[p][t][I + i] (slice order), rounded to BF16.
__global__ void __launch_bounds__(256)
    swiglu_reduce_kernel(const float* __restrict__ parts, int n_parts, int T, int I, float limit,
                         __nv_bfloat16* __restrict__ h) {
  const size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= static_cast<size_t>(T) * I) return;
  const size_t t = i / I, c = i % I;
  float g = 0.f, u = 0.f;
  for (int p = 0; p < n_parts; ++p) {
    const float* row = parts + (static_cast<size_t>(p) * T + t) * 2 * I;
    g += __ldg(row + c);
    u += __ldg(row + I + c);
  }
  h[i] = __float2bfloat16_rn(clamped_swiglu_f32(g, u, limit));
}

// W13 layout: for each group g and 128-row tile mt of the expert width, 256
// consecutive rows = W1[g][mt*128 .. +128) followed by W3[g][mt*128 .. +128),
// so one TMA box of 256 rows feeds both gate and up MMAs of a tile.
__global__ void __launch_bounds__(256)
    repack_w13_kernel(const uint4* __restrict__ w1, const uint4* __restrict__ w3, const uint4* __restrict__ sh1,
                      const uint4* __restrict__ sh3, int E, int S, int I, int hv, uint4* __restrict__ dst) {
  const size_t row = static_cast<size_t>(blockIdx.x) * 8 + threadIdx.x / 32;
  const size_t total = static_cast<size_t>(E + S) * 2 * I;
  if (row >= total) return;
  const int g = static_cast<int>(row / (2 * I));
  const int rr = static_cast<int>(row % (2 * I));
  const int mt = rr / 256, within = rr % 256;
  const int src_row = mt * 128 + (within & 127);
  const bool up = within >= 128;
  const uint4* base = g < E ? (up ? w3 : w1) + static_cast<size_t>(g) * I * hv
                            : (up ? sh3 : sh1) + static_cast<size_t>(g - E) * I * hv;
  const uint4* src = base + static_cast<size_t>(src_row) * hv;
  uint4* d = dst + row * hv;
  for (int c = threadIdx.x % 32; c < hv; c += 32) d[c] = __ldg(src + c);
}

// Scale atoms of the block-scaled MMA: for each group, 128-row weight tile and
// 128-wide K block, 512 bytes holding row m, block kb at (m % 32) * 16 +
// (m / 32) * 4 + kb (rows interleaved by 32 so that a 32-lane x 16-byte copy
// to TMEM puts every row's four scales in one 32-bit word). With two sources
// (W1, W3) the two atoms of the same rows are adjacent.
__global__ void __launch_bounds__(256)
    sf_atoms_kernel(const uint8_t* __restrict__ sa, const uint8_t* __restrict__ sb, int groups, int rows, int K,
                    uint8_t* __restrict__ dst, int* bad) {
  const int parts = sb ? 2 : 1;
  const int mtiles = rows / 128, kb4s = K / 128;
  const size_t total = static_cast<size_t>(groups) * mtiles * kb4s * parts * 512;
  const size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= total) return;
  const int within = static_cast<int>(i % 512);
  size_t rest = i / 512;
  const int p = static_cast<int>(rest % parts);
  rest /= parts;
  const int kb4 = static_cast<int>(rest % kb4s);
  rest /= kb4s;
  const int mt = static_cast<int>(rest % mtiles);
  const size_t g = rest / mtiles;
  const int rem = within % 16;
  const int m = mt * 128 + (rem / 4) * 32 + within / 16;
  const int kblk = kb4 * 4 + rem % 4;
  const uint8_t v = (p ? sb : sa)[(g * rows + m) * (K / 32) + kblk];
  if (v == 0xFF) atomicOr(bad, 1);
  dst[i] = v;
}

// One thread per 32-element block: OCP MX rule with E2M1 elements.
__global__ void __launch_bounds__(256)
    quantize_mxfp4_kernel(const uint4* __restrict__ src, int64_t nblocks, uint4* __restrict__ packed,
                          uint8_t* __restrict__ scales) {
  const int64_t b = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (b >= nblocks) return;
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
  int code = 0;
  float inv_scale = 0.f;
  if (amax > 0.f) {
    int ex;
    frexpf(amax, &ex);                       // amax = f * 2^ex, f in [0.5, 1)
    int shared = (ex - 1) - 2;               // floor(log2(amax)) - emax(E2M1)
    shared = max(-127, min(127, shared));
    code = shared + 127;
    inv_scale = ldexpf(1.0f, -shared);       // exact power of two
  }
  uint32_t words[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const float q = v[i] * inv_scale;
    const float a = fabsf(q);
    // nearest E2M1 magnitude, ties to the even code, saturating at 6
    const uint32_t mag = (a > 0.25f) + (a >= 0.75f) + (a > 1.25f) + (a >= 1.75f) + (a > 2.5f) + (a >= 3.5f) + (a > 5.0f);
    const uint32_t c = mag | (signbit(q) ? 8u : 0u);
    words[i / 8] |= c << (4 * (i % 8));
  }
  packed[b] = make_uint4(words[0], words[1], words[2], words[3]);
  scales[b] = static_cast<uint8_t>(code);
}

// One thread per 32-element block: OCP MX rule with E4M3 elements (MXFP8), the
// same rule the activations use, conversion rounding to nearest-even and
// saturating at +-448.
__global__ void __launch_bounds__(256)
    quantize_mxfp8_kernel(const uint4* __restrict__ src, int64_t nblocks, uint4* __restrict__ codes,
                          uint8_t* __restrict__ scales) {
  const int64_t b = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (b >= nblocks) return;
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
  codes[b * 2] = make_uint4(w[0], w[1], w[2], w[3]);
  codes[b * 2 + 1] = make_uint4(w[4], w[5], w[6], w[7]);
  scales[b] = static_cast<uint8_t>(code);
}

// Read-only streaming: one thread per CTA keeps kReadStages bulk copies of
// kReadChunk bytes (global -> this CTA's shared memory) in flight over its
// chunks (every gridDim-th one), the way the GEMMs' producers stream weights,
// and computes nothing. Waits are bounded; a wait that runs out sets the status.
constexpr int kReadStages = 6;
constexpr int kReadChunk = 32 * 1024;

__global__ void __launch_bounds__(32)
    stream_read_kernel(const uint8_t* __restrict__ buf, long nchunks, int* status,
                       unsigned long long timeout_ns) {
  extern __shared__ __align__(1024) uint8_t ring[];
  __shared__ uint64_t bar[kReadStages];
  if (threadIdx.x != 0) return;
  for (int i = 0; i < kReadStages; ++i) mbar_init(&bar[i], 1);
  fence_mbarrier_init();
  long next = blockIdx.x;
  long issued = 0;
  for (int i = 0; i < kReadStages && next < nchunks; ++i, next += gridDim.x, ++issued) {
    mbar_arrive_expect_tx(&bar[i], kReadChunk);
    bulk_load(ring + i * kReadChunk, buf + next * kReadChunk, kReadChunk, &bar[i], kCacheEvictFirst);
  }
  for (long done = 0; done < issued; ++done) {
    const int st = static_cast<int>(done % kReadStages);
    if (!mbar_wait(&bar[st], static_cast<uint32_t>((done / kReadStages) & 1), timeout_ns)) {
      report_status(status, kStatusTimeout);
      // let the copies still in flight land before the CTA exits
      for (long j = done + 1; j < issued; ++j)
        mbar_wait(&bar[j % kReadStages], static_cast<uint32_t>((j / kReadStages) & 1), timeout_ns);
      return;
    }
    if (next < nchunks) {
      mbar_arrive_expect_tx(&bar[st], kReadChunk);
      bulk_load(ring + st * kReadChunk, buf + next * kReadChunk, kReadChunk, &bar[st], kCacheEvictFirst);
      next += gridDim.x;
      ++issued;
    }
  }
}

__global__ void wait_timeout_probe_kernel(int* status, unsigned long long timeout_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbarrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // Nothing ever arrives on `bar`: the wait must run out and report.
    if (!mbar_wait(&bar, 0, timeout_ns)) report_status(status, kStatusTimeout);
  }
  __syncthreads();
}

}  // namespace

cudaError_t launch_combine(const float* O, const int32_t* inv, const int32_t* idx, int e_begin, int e_count,
                           const float* w, int T, int H, int k, int S, void* y, bool y_f32, const float* sh_parts,
                           int n_parts, cudaStream_t s) {
  if (T == 0) return cudaSuccess;
  if (k > kCombineMaxK) return cudaErrorInvalidValue;
  const int H4 = H / 4;
  const dim3 grid(T, (H4 + 127) / 128);
  combine_kernel<<<grid, 128, 0, s>>>(reinterpret_cast<const float4*>(O), inv, idx, e_begin, e_count, w, T, H4, k,
                                      S, y, y_f32 ? 1 : 0, reinterpret_cast<const float4*>(sh_parts), n_parts);
  return cudaGetLastError();
}

cudaError_t launch_swiglu_reduce(const float* parts, int n_parts, int T, int I, float limit, void* h,
                                 cudaStream_t s) {
  const size_t n = static_cast<size_t>(T) * I;
  if (n == 0) return cudaSuccess;
  swiglu_reduce_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(parts, n_parts, T, I, limit,
                                                                             static_cast<__nv_bfloat16*>(h));
  return cudaGetLastError();
}

cudaError_t launch_repack_w13_bytes(const void* w1, const void* w3, const void* sh1, const void* sh3, int E, int S,
                                    int I, int row_bytes, void* w13, cudaStream_t s) {
  const size_t rows = static_cast<size_t>(E + S) * 2 * I;
  if (rows == 0) return cudaSuccess;
  repack_w13_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, s>>>(
      static_cast<const uint4*>(w1), static_cast<const uint4*>(w3), static_cast<const uint4*>(sh1),
      static_cast<const uint4*>(sh3), E, S, I, row_bytes / 16, static_cast<uint4*>(w13));
  return cudaGetLastError();
}

cudaError_t launch_repack_w13(const void* w1, const void* w3, const void* sh1, const void* sh3, int E, int S, int I,
                              int H, void* w13, cudaStream_t s) {
  return launch_repack_w13_bytes(w1, w3, sh1, sh3, E, S, I, H * 2, w13, s);
}

cudaError_t launch_sf_atoms(const uint8_t* s_a, const uint8_t* s_b, int groups, int rows, int K, uint8_t* dst,
                            int* bad, cudaStream_t s) {
  const size_t total = static_cast<size_t>(groups) * (rows / 128) * (K / 128) * (s_b ? 2 : 1) * 512;
  if (total == 0) return cudaSuccess;
  sf_atoms_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, s>>>(s_a, s_b, groups, rows, K, dst, bad);
  return cudaGetLastError();
}

cudaError_t launch_quantize_mxfp4(const void* src, int64_t rows, int cols, uint8_t* packed, uint8_t* scales,
                                  cudaStream_t s) {
  const int64_t nblocks = rows * (cols / 32);
  if (nblocks == 0) return cudaSuccess;
  quantize_mxfp4_kernel<<<static_cast<unsigned>((nblocks + 255) / 256), 256, 0, s>>>(
      static_cast<const uint4*>(src), nblocks, reinterpret_cast<uint4*>(packed), scales);
  return cudaGetLastError();
}

cudaError_t launch_quantize_mxfp8(const void* src, int64_t rows, int cols, uint8_t* codes, uint8_t* scales,
                                  cudaStream_t s) {
  const int64_t nblocks = rows * (cols / 32);
  if (nblocks == 0) return cudaSuccess;
  quantize_mxfp8_kernel<<<static_cast<unsigned>((nblocks + 255) / 256), 256, 0, s>>>(
      static_cast<const uint4*>(src), nblocks, reinterpret_cast<uint4*>(codes), scales);
  return cudaGetLastError();
}

cudaError_t launch_stream_read(const void* buf, size_t bytes, int grid, int* status, unsigned long long timeout_ns,
                               cudaStream_t s) {
  const long nchunks = static_cast<long>(bytes / kReadChunk);
  if (nchunks == 0) return cudaSuccess;
  const int smem = kReadStages * kReadChunk;
  cudaError_t e = cudaFuncSetAttribute(stream_read_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  stream_read_kernel<<<grid, 32, smem, s>>>(static_cast<const uint8_t*>(buf), nchunks, status, timeout_ns);
  return cudaGetLastError();
}

cudaError_t launch_wait_timeout_probe(int* status, unsigned long long timeout_ns, cudaStream_t s) {
  wait_timeout_probe_kernel<<<1, 32, 0, s>>>(status, timeout_ns);
  return cudaGetLastError();
}

}  // namespace moe
