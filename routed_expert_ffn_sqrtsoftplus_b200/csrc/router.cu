// Router: logits, sqrtsoftplus scores, top-k selection and weight normalisation.
//
// DeepSeek V4.1 inference/config.json: "score_func": "sqrtsoftplus",
// "n_activated_experts": 6, "route_scale": 1.5. Computed as
//   z_e = x . Wg_e + b_e,  s_e = sqrt(softplus(z_e)),
//   top-k by s (ties: lower expert index), w_j = route_scale * s_j / sum_sel s.
//
// Two stages:
//  1. approximate fp32 logits for all experts (CUDA cores here for small T, or
//     the tcgen05 GEMM in dense mode for large T);
//  2. one warp per token: fp32 scores from the approximate logits, the k-th
//     largest score s_k, and a candidate set {e : s_e >= s_k - delta}. Every
//     candidate's logit is recomputed exactly (BF16 x BF16 products are exact
//     in fp32; they are summed in fp64) and the scores, the selection and the
//     weights are taken from these fp64 values. With |approx error| < delta/2
//     no expert outside the candidate set can belong to the true top-k, so the
//     selection equals the exact one except on genuine fp64-level ties.
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kLogitWarps = 8;     // experts per CTA (one per warp)
constexpr int kLogitTokens = 64;   // tokens per CTA
constexpr int kTokPerPass = 4;     // tokens a warp accumulates at once

__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float (&f)[8]) {
  const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 t = __bfloat1622float2(p[i]);
    f[2 * i] = t.x;
    f[2 * i + 1] = t.y;
  }
}

// z[t, e] = sum_h x[t, h] * wg[e, h] (+ bias[e]); fp32 accumulation per lane,
// then a warp tree sum.
__global__ void __launch_bounds__(kLogitWarps * 32)
    router_logits_kernel(const uint4* __restrict__ x, const uint4* __restrict__ wg, const float* __restrict__ bias,
                         float* __restrict__ z, int T, int H, int E) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int e = blockIdx.x * kLogitWarps + warp;
  if (e >= E) return;
  const int hv = H / 8;  // uint4 chunks per row
  const uint4* wrow = wg + static_cast<size_t>(e) * hv;
  const float b = bias ? bias[e] : 0.0f;
  const int t_begin = blockIdx.y * kLogitTokens;
  const int t_end = min(T, t_begin + kLogitTokens);
  for (int t0 = t_begin; t0 < t_end; t0 += kTokPerPass) {
    float acc[kTokPerPass] = {0.f, 0.f, 0.f, 0.f};
    for (int c = lane; c < hv; c += 32) {
      float wf[8];
      bf16x8_to_f32(__ldg(wrow + c), wf);
#pragma unroll
      for (int tt = 0; tt < kTokPerPass; ++tt) {
        if (t0 + tt < t_end) {
          float xf[8];
          bf16x8_to_f32(__ldg(x + static_cast<size_t>(t0 + tt) * hv + c), xf);
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[tt] = fmaf(xf[i], wf[i], acc[tt]);
        }
      }
    }
#pragma unroll
    for (int tt = 0; tt < kTokPerPass; ++tt) {
      float v = acc[tt];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0 && t0 + tt < t_end) z[static_cast<size_t>(t0 + tt) * E + e] = v + b;
    }
  }
}

// Approximate logits for up to 32 tokens: CTA = 8 experts x one slice of P
// hidden values (the tokens' slice staged in shared memory), one warp per
// expert, 32 fp32 partial sums per lane reduced with a halving butterfly
// (31 shuffles leave token l's sum in lane l). Slices are written separately
// ([slice][T][E]) and summed in slice order by the top-k kernel.
constexpr int kSmallTok = 32;
constexpr int kSmallMaxSlice = 1024;                            // P <= 1024
constexpr int kSmallWChunks = kSmallMaxSlice / 8 / 32;          // Wg chunks per lane
constexpr int kSmallStage = kSmallTok * kSmallMaxSlice / 8 / 256;  // x chunks per thread

__global__ void __launch_bounds__(256)
    router_small_kernel(const uint4* __restrict__ x, const uint4* __restrict__ wg, float* __restrict__ part, int T,
                        int H, int E, int P) {
  extern __shared__ uint4 xs[];  // [T][P / 8]
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int slice = blockIdx.y;
  const int pv = P / 8, hv = H / 8;
  const int e = blockIdx.x * 8 + warp;
  const uint4* wrow = wg + static_cast<size_t>(e < E ? e : 0) * hv + slice * pv;
  // this lane's Wg chunks (pv <= 128: at most 4), issued before the x staging so
  // both sets of loads are in flight together
  uint4 wv[kSmallWChunks];
#pragma unroll
  for (int j = 0; j < kSmallWChunks; ++j)
    if (lane + 32 * j < pv) wv[j] = __ldg(wrow + lane + 32 * j);
  // stage the tokens' slice: every load of a thread issued before its stores
  const int n = T * pv;
  {
    uint4 tmp[kSmallStage];
#pragma unroll
    for (int j = 0; j < kSmallStage; ++j) {
      const int i = threadIdx.x + j * 256;
      if (i < n) tmp[j] = __ldg(x + static_cast<size_t>(i / pv) * hv + slice * pv + i % pv);
    }
#pragma unroll
    for (int j = 0; j < kSmallStage; ++j) {
      const int i = threadIdx.x + j * 256;
      if (i < n) xs[i] = tmp[j];
    }
  }
  __syncthreads();
  if (e >= E) return;
  float v[kSmallTok];
#pragma unroll
  for (int i = 0; i < kSmallTok; ++i) v[i] = 0.f;
#pragma unroll
  for (int j = 0; j < kSmallWChunks; ++j) {
    const int c = lane + 32 * j;
    if (c >= pv) break;
    float wf[8];
    bf16x8_to_f32(wv[j], wf);
#pragma unroll
    for (int tt = 0; tt < kSmallTok; ++tt) {
      if (tt < T) {
        float xf[8];
        bf16x8_to_f32(xs[tt * pv + c], xf);
#pragma unroll
        for (int i = 0; i < 8; ++i) v[tt] = fmaf(xf[i], wf[i], v[tt]);
      }
    }
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < o; ++i) {
      const float send = upper ? v[i] : v[i + o];
      const float keep = upper ? v[i + o] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  if (lane < T) part[(static_cast<size_t>(slice) * T + lane) * E + e] = v[0];
}

__device__ __forceinline__ float softplus_f32(float z) { return fmaxf(z, 0.0f) + log1pf(expf(-fabsf(z))); }
__device__ __forceinline__ double softplus_f64(double z) { return fmax(z, 0.0) + log1p(exp(-fabs(z))); }

// Warp-wide argmax over (value desc, index asc). Returns the winner on all lanes.
__device__ __forceinline__ void warp_argmax(float& v, int& i) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, v, o);
    const int oi = __shfl_xor_sync(0xffffffffu, i, o);
    if (ov > v || (ov == v && oi < i)) {
      v = ov;
      i = oi;
    }
  }
}
__device__ __forceinline__ void warp_argmax_d(double& v, int& i) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const double ov = __shfl_xor_sync(0xffffffffu, v, o);
    const int oi = __shfl_xor_sync(0xffffffffu, i, o);
    if (ov > v || (ov == v && oi < i)) {
      v = ov;
      i = oi;
    }
  }
}

// Writes one token's selection. A token whose scores are not finite numbers
// (NaN or infinite x, router weights or bias) can leave a selection slot
// without a valid expert; such a slot gets expert r (an in-range placeholder,
// so the permutation and the combine never index outside their buffers) and a
// NaN weight, which makes the token's output NaN, and the device status word
// records MOE_ERR_DEVICE.
__device__ __forceinline__ void write_selection(const int* sel_e, const double* sel_s, double sum, int k, int E,
                                                float route_scale, int32_t* idx, float* w, int* status) {
  for (int r = 0; r < k; ++r) {
    int e = sel_e[r];
    float wr = static_cast<float>(route_scale * (sel_s[r] / sum));
    if (e < 0 || e >= E) {
      report_status(status, kStatusDevice);
      e = r;
      wr = __int_as_float(0x7fc00000);
    }
    idx[r] = e;
    w[r] = wr;
  }
}

constexpr int kTopkWarps = 8;
constexpr int kPartBatch = 4;      // logit slices loaded together (top-k CTA kernel)
constexpr int kWBatch = 10;        // Wg chunks per lane loaded together (exact re-scoring)
constexpr int kMaxCand = 64;       // candidates refined per token
constexpr int kMaxEPL = 16;        // experts per lane (E <= 512)
constexpr int kMaxK = 32;

template <int EPL>
__global__ void __launch_bounds__(kTopkWarps * 32)
    topk_refine_kernel(const float* __restrict__ z, const uint4* __restrict__ x, const uint4* __restrict__ wg,
                       const float* __restrict__ bias, int T, int H, int E, int k, float route_scale, float delta,
                       int32_t* __restrict__ idx_out, float* __restrict__ w_out, int* status) {
  __shared__ int cand_s[kTopkWarps][kMaxCand];
  __shared__ double cs_s[kTopkWarps][kMaxCand];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int t = blockIdx.x * kTopkWarps + warp;
  if (t >= T) return;
  int* cand = cand_s[warp];
  double* cs = cs_s[warp];

  // 1. approximate scores
  float s[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    const int e = lane + 32 * i;
    s[i] = e < E ? sqrtf(softplus_f32(z[static_cast<size_t>(t) * E + e])) : -INFINITY;
  }
  // 2. k-th largest approximate score
  float kth = 0.f;
  {
    float tmp[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) tmp[i] = s[i];
    for (int r = 0; r < k; ++r) {
      float bv = -INFINITY;
      int bi = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        if (tmp[i] > bv || (tmp[i] == bv && e < bi)) {
          bv = tmp[i];
          bi = e;
        }
      }
      warp_argmax(bv, bi);
      kth = bv;
#pragma unroll
      for (int i = 0; i < EPL; ++i)
        if (lane + 32 * i == bi) tmp[i] = -INFINITY;
    }
  }
  // 3. candidates in ascending expert order
  const float thr = kth - delta;
  int ncand = 0;
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    const bool f = s[i] >= thr;
    const unsigned m = __ballot_sync(0xffffffffu, f);
    const int pos = ncand + __popc(m & ((1u << lane) - 1u));
    if (f && pos < kMaxCand) cand[pos] = lane + 32 * i;
    ncand += __popc(m);
  }
  if (ncand > kMaxCand) {
    // Degenerate router (more than kMaxCand experts within delta of the k-th
    // score): keep the kMaxCand best by approximate score, lower index first.
    float tmp[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) tmp[i] = s[i];
    for (int r = 0; r < kMaxCand; ++r) {
      float bv = -INFINITY;
      int bi = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        if (tmp[i] > bv || (tmp[i] == bv && e < bi)) {
          bv = tmp[i];
          bi = e;
        }
      }
      warp_argmax(bv, bi);
      if (lane == 0) cand[r] = bi;
#pragma unroll
      for (int i = 0; i < EPL; ++i)
        if (lane + 32 * i == bi) tmp[i] = -INFINITY;
    }
    ncand = kMaxCand;
  }
  __syncwarp();

  // 4. exact logits of the candidates: fp32 products (exact), fp64 sums
  const int hv = H / 8;
  const uint4* xrow = x + static_cast<size_t>(t) * hv;
  for (int c = 0; c < ncand; ++c) {
    const int e = cand[c];
    const uint4* wrow = wg + static_cast<size_t>(e) * hv;
    double acc = 0.0;
    for (int j = lane; j < hv; j += 32) {
      float xf[8], wf[8];
      bf16x8_to_f32(__ldg(xrow + j), xf);
      bf16x8_to_f32(__ldg(wrow + j), wf);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc += static_cast<double>(xf[i] * wf[i]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
      const double zz = acc + (bias ? static_cast<double>(bias[e]) : 0.0);
      cs[c] = sqrt(softplus_f64(zz));
    }
  }
  __syncwarp();

  // 5. exact top-k among the candidates, then the weights
  double v0 = lane < ncand ? cs[lane] : -INFINITY;
  double v1 = lane + 32 < ncand ? cs[lane + 32] : -INFINITY;
  const int e0 = lane < ncand ? cand[lane] : 0x7fffffff;
  const int e1 = lane + 32 < ncand ? cand[lane + 32] : 0x7fffffff;
  double sel_s[kMaxK];
  int sel_e[kMaxK];
  double sum = 0.0;
  for (int r = 0; r < k; ++r) {
    double bv;
    int bi;
    if (v0 > v1 || (v0 == v1 && e0 < e1)) {
      bv = v0;
      bi = e0;
    } else {
      bv = v1;
      bi = e1;
    }
    warp_argmax_d(bv, bi);
    if (e0 == bi) v0 = -INFINITY;
    if (e1 == bi) v1 = -INFINITY;
    sel_s[r] = bv;
    sel_e[r] = bi;
    sum += bv;
  }
  if (lane == 0) write_selection(sel_e, sel_s, sum, k, E, route_scale, idx_out + static_cast<size_t>(t) * k,
                                  w_out + static_cast<size_t>(t) * k, status);
}

// Top-k for few tokens, one CTA per token: warp 0 forms the approximate scores
// (sum of the logit slices + bias), the k-th score and the candidate set
// {s >= s_k - delta}; the 8 warps then re-score the candidates exactly (fp32
// products, fp64 sums, four independent accumulators per lane) in parallel,
// and warp 0 takes the top-k of the exact scores and the weights.
// `bias` is added to the summed slices (pass nullptr when the logits already hold
// it); `exact_bias` is the bias of the exact re-scoring.
template <int EPL>
__global__ void __launch_bounds__(256)
    topk_cta_kernel(const float* __restrict__ part, int nparts, const uint4* __restrict__ x,
                    const uint4* __restrict__ wg, const float* __restrict__ bias, int T, int H, int E, int k,
                    float route_scale, float delta, int32_t* __restrict__ idx_out, float* __restrict__ w_out,
                    float* __restrict__ z_out, int* status, const float* __restrict__ exact_bias) {
  __shared__ int cand[kMaxCand];
  __shared__ double cs[kMaxCand];
  __shared__ int ncand_s;
  extern __shared__ uint4 xrow_s[];  // this token's row (H / 8 chunks), staged by warps 1..7
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int t = blockIdx.x;
  const int hv = H / 8;
  const uint4* xrow = x + static_cast<size_t>(t) * hv;
  if (warp != 0) {
    for (int c = threadIdx.x - 32; c < hv; c += blockDim.x - 32) xrow_s[c] = __ldg(xrow + c);
  } else {
    // summed logit slices, added in slice order; all of a lane's loads are
    // independent, so they are issued together
    float s[EPL];
    float zi[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      zi[i] = (e < E && bias) ? bias[e] : 0.f;
    }
    int p = 0;
    for (; p + kPartBatch <= nparts; p += kPartBatch) {
      float pv[kPartBatch][EPL];
#pragma unroll
      for (int q = 0; q < kPartBatch; ++q)
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
          const int e = lane + 32 * i;
          pv[q][i] = e < E ? part[(static_cast<size_t>(p + q) * T + t) * E + e] : 0.f;
        }
#pragma unroll
      for (int q = 0; q < kPartBatch; ++q)
#pragma unroll
        for (int i = 0; i < EPL; ++i) zi[i] += pv[q][i];
    }
    for (; p < nparts; ++p)
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        const int e = lane + 32 * i;
        if (e < E) zi[i] += part[(static_cast<size_t>(p) * T + t) * E + e];
      }
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      if (e < E) {
        if (z_out) z_out[static_cast<size_t>(t) * E + e] = zi[i];
        s[i] = sqrtf(softplus_f32(zi[i]));
      } else {
        s[i] = -INFINITY;
      }
    }
    float kth = 0.f;
    {
      float tmp[EPL];
#pragma unroll
      for (int i = 0; i < EPL; ++i) tmp[i] = s[i];
      for (int r = 0; r < k; ++r) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
          const int e = lane + 32 * i;
          if (tmp[i] > bv || (tmp[i] == bv && e < bi)) {
            bv = tmp[i];
            bi = e;
          }
        }
        warp_argmax(bv, bi);
        kth = bv;
#pragma unroll
        for (int i = 0; i < EPL; ++i)
          if (lane + 32 * i == bi) tmp[i] = -INFINITY;
      }
    }
    const float thr = kth - delta;
    int n = 0;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const bool f = s[i] >= thr;
      const unsigned m = __ballot_sync(0xffffffffu, f);
      const int pos = n + __popc(m & ((1u << lane) - 1u));
      if (f && pos < kMaxCand) cand[pos] = lane + 32 * i;
      n += __popc(m);
    }
    if (n > kMaxCand) {
      float tmp[EPL];
#pragma unroll
      for (int i = 0; i < EPL; ++i) tmp[i] = s[i];
      for (int r = 0; r < kMaxCand; ++r) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
          const int e = lane + 32 * i;
          if (tmp[i] > bv || (tmp[i] == bv && e < bi)) {
            bv = tmp[i];
            bi = e;
          }
        }
        warp_argmax(bv, bi);
        if (lane == 0) cand[r] = bi;
#pragma unroll
        for (int i = 0; i < EPL; ++i)
          if (lane + 32 * i == bi) tmp[i] = -INFINITY;
      }
      n = kMaxCand;
    }
    if (lane == 0) ncand_s = n;
  }
  __syncthreads();
  const int ncand = ncand_s;
  for (int c = warp; c < ncand; c += 8) {
    const int e = cand[c];
    const uint4* wrow = wg + static_cast<size_t>(e) * hv;
    // chunk q of this lane is j = lane + 32 q; four accumulators by q mod 4, each
    // in increasing q; the Wg chunks of a batch are loaded together
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    const int nq = (hv - lane + 31) / 32;
    for (int q0 = 0; q0 < nq; q0 += kWBatch) {
      uint4 wv[kWBatch];
#pragma unroll
      for (int u = 0; u < kWBatch; ++u)
        if (q0 + u < nq) wv[u] = __ldg(wrow + lane + 32 * (q0 + u));
#pragma unroll
      for (int u = 0; u < kWBatch; ++u) {
        if (q0 + u < nq) {
          float xf[8], wf[8];
          bf16x8_to_f32(xrow_s[lane + 32 * (q0 + u)], xf);
          bf16x8_to_f32(wv[u], wf);
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[(q0 + u) & 3] += static_cast<double>(xf[i] * wf[i]);
        }
      }
    }
    double a = (acc[0] + acc[1]) + (acc[2] + acc[3]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
    if (lane == 0) cs[c] = sqrt(softplus_f64(a + (exact_bias ? static_cast<double>(exact_bias[e]) : 0.0)));
  }
  __syncthreads();
  if (warp != 0) return;
  double v0 = lane < ncand ? cs[lane] : -INFINITY;
  double v1 = lane + 32 < ncand ? cs[lane + 32] : -INFINITY;
  const int e0 = lane < ncand ? cand[lane] : 0x7fffffff;
  const int e1 = lane + 32 < ncand ? cand[lane + 32] : 0x7fffffff;
  double sel_s[kMaxK];
  int sel_e[kMaxK];
  double sum = 0.0;
  for (int r = 0; r < k; ++r) {
    double bv;
    int bi;
    if (v0 > v1 || (v0 == v1 && e0 < e1)) {
      bv = v0;
      bi = e0;
    } else {
      bv = v1;
      bi = e1;
    }
    warp_argmax_d(bv, bi);
    if (e0 == bi) v0 = -INFINITY;
    if (e1 == bi) v1 = -INFINITY;
    sel_s[r] = bv;
    sel_e[r] = bi;
    sum += bv;
  }
  if (lane == 0) write_selection(sel_e, sel_s, sum, k, E, route_scale, idx_out + static_cast<size_t>(t) * k,
                                  w_out + static_cast<size_t>(t) * k, status);
}

// Hash-routed layers (MAX DeepseekV41Config num_hash_layers): token t takes the
// k experts of row ids[t] of the layer's table, in the table's order; their
// weights are the sqrtsoftplus scores normalised over the k and scaled by
// route_scale. One CTA per token: warp j re-scores experts j, j + 8, ... exactly
// (fp32-exact BF16 products, fp64 sums, as the learned routing's refinement),
// warp 0 normalises. An id outside [0, vocab) gives the placeholder experts
// 0..k-1 with NaN weights and records a device error.
__global__ void __launch_bounds__(256)
    hash_route_kernel(const uint4* __restrict__ x, const uint4* __restrict__ wg, const float* __restrict__ bias,
                      const int32_t* __restrict__ table, const int32_t* __restrict__ ids, int H, int E, int k,
                      int vocab, float route_scale, int32_t* __restrict__ idx_out, float* __restrict__ w_out,
                      int* status) {
  __shared__ double sc[kMaxK];
  __shared__ int ex[kMaxK];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int t = blockIdx.x;
  const int id = ids[t];
  const bool ok = id >= 0 && id < vocab;
  const int hv = H / 8;
  const uint4* xrow = x + static_cast<size_t>(t) * hv;
  for (int j = warp; j < k; j += 8) {
    const int e = ok ? table[static_cast<size_t>(id) * k + j] : j;
    const uint4* wrow = wg + static_cast<size_t>(e) * hv;
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    for (int c = lane, q = 0; c < hv; c += 32, ++q) {
      float xf[8], wf[8];
      bf16x8_to_f32(__ldg(xrow + c), xf);
      bf16x8_to_f32(__ldg(wrow + c), wf);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[q & 3] += static_cast<double>(xf[i] * wf[i]);
    }
    double a = (acc[0] + acc[1]) + (acc[2] + acc[3]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
    if (lane == 0) {
      sc[j] = sqrt(softplus_f64(a + (bias ? static_cast<double>(bias[e]) : 0.0)));
      ex[j] = e;
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (!ok) report_status(status, kStatusDevice);
    double sum = 0.0;
    for (int j = 0; j < k; ++j) sum += sc[j];
    for (int j = 0; j < k; ++j) {
      idx_out[static_cast<size_t>(t) * k + j] = ex[j];
      w_out[static_cast<size_t>(t) * k + j] =
          ok ? static_cast<float>(route_scale * (sc[j] / sum)) : __int_as_float(0x7fc00000);
    }
  }
}

// Table check: every entry in [0, E) and no expert twice in a row.
__global__ void __launch_bounds__(256)
    hash_table_check_kernel(const int32_t* __restrict__ table, int vocab, int k, int E, int* bad) {
  const int v = blockIdx.x * blockDim.x + threadIdx.x;
  if (v >= vocab) return;
  const int32_t* row = table + static_cast<size_t>(v) * k;
  for (int j = 0; j < k; ++j) {
    const int e = row[j];
    if (e < 0 || e >= E) {
      atomicOr(bad, 1);
      return;
    }
    for (int i = 0; i < j; ++i)
      if (row[i] == e) {
        atomicOr(bad, 1);
        return;
      }
  }
}

}  // namespace

cudaError_t launch_hash_route(const void* x, const void* wg, const float* bias, const int32_t* table,
                              const int32_t* ids, int T, int H, int E, int k, int vocab, float route_scale,
                              int32_t* idx, float* w, int* status, cudaStream_t s) {
  if (k > kMaxK || T == 0) return T == 0 ? cudaSuccess : cudaErrorInvalidValue;
  hash_route_kernel<<<T, 256, 0, s>>>(static_cast<const uint4*>(x), static_cast<const uint4*>(wg), bias, table, ids,
                                      H, E, k, vocab, route_scale, idx, w, status);
  return cudaGetLastError();
}

cudaError_t launch_hash_table_check(const int32_t* table, int vocab, int k, int E, int* bad, cudaStream_t s) {
  hash_table_check_kernel<<<(vocab + 255) / 256, 256, 0, s>>>(table, vocab, k, E, bad);
  return cudaGetLastError();
}

cudaError_t router_set_attributes() {
  return cudaFuncSetAttribute(router_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmallTok * 1024 * 2);
}

int router_small_slice(int H) {
  for (int p : {1024, 512, 256, 128})
    if (H % p == 0) return p;
  return 0;
}

cudaError_t launch_router_small(const void* x, const void* wg, float* part, int T, int H, int E, cudaStream_t s) {
  const int P = router_small_slice(H);
  if (P == 0 || T > kSmallTok) return cudaErrorInvalidValue;
  const size_t smem = static_cast<size_t>(T) * P * 2;
  const dim3 grid((E + 7) / 8, H / P);
  router_small_kernel<<<grid, 256, smem, s>>>(static_cast<const uint4*>(x), static_cast<const uint4*>(wg), part, T,
                                              H, E, P);
  return cudaGetLastError();
}

cudaError_t launch_topk_small(const float* part, int nparts, const void* x, const void* wg, const float* bias, int T,
                              int H, int E, int k, float route_scale, float delta, int32_t* idx, float* w, float* z,
                              int* status, cudaStream_t s, const float* exact_bias) {
  // the token's row is staged in shared memory (within the default 48 KB)
  if (k > kMaxK || E > 32 * kMaxEPL || static_cast<size_t>(H) * 2 > 40 * 1024) return cudaErrorInvalidValue;
  const uint4* xv = static_cast<const uint4*>(x);
  const uint4* wv = static_cast<const uint4*>(wg);
  const int epl = (E + 31) / 32;
#define MOE_TOPKS_CASE(N)                                                                                      \
  if (epl <= N) {                                                                                              \
    topk_cta_kernel<N><<<T, 256, static_cast<size_t>(H) * 2, s>>>(part, nparts, xv, wv, bias, T, H, E, k,      \
                                                                 route_scale, delta, idx, w, z,                  \
                                         status, exact_bias);                                                  \
    return cudaGetLastError();                                                                                 \
  }
  MOE_TOPKS_CASE(1)
  MOE_TOPKS_CASE(4)
  MOE_TOPKS_CASE(12)
  MOE_TOPKS_CASE(16)
#undef MOE_TOPKS_CASE
  return cudaErrorInvalidValue;
}

cudaError_t launch_router_logits(const void* x, const void* wg, const float* bias, float* z, int T, int H, int E,
                                 cudaStream_t s) {
  dim3 grid((E + kLogitWarps - 1) / kLogitWarps, (T + kLogitTokens - 1) / kLogitTokens);
  router_logits_kernel<<<grid, kLogitWarps * 32, 0, s>>>(static_cast<const uint4*>(x), static_cast<const uint4*>(wg),
                                                         bias, z, T, H, E);
  return cudaGetLastError();
}

cudaError_t launch_topk_refine(const float* z, const void* x, const void* wg, const float* bias, int T, int H,
                               int E, int k, float route_scale, float delta, int32_t* idx, float* w, int* status,
                               cudaStream_t s) {
  if (k > kMaxK || E > 32 * kMaxEPL) return cudaErrorInvalidValue;
  const dim3 grid((T + kTopkWarps - 1) / kTopkWarps);
  const uint4* xv = static_cast<const uint4*>(x);
  const uint4* wv = static_cast<const uint4*>(wg);
  const int epl = (E + 31) / 32;
#define MOE_TOPK_CASE(N)                                                                                 \
  if (epl <= N) {                                                                                        \
    topk_refine_kernel<N><<<grid, kTopkWarps * 32, 0, s>>>(z, xv, wv, bias, T, H, E, k, route_scale, delta, \
                                                           idx, w, status);                              \
    return cudaGetLastError();                                                                           \
  }
  MOE_TOPK_CASE(1)
  MOE_TOPK_CASE(4)
  MOE_TOPK_CASE(12)
  MOE_TOPK_CASE(16)
#undef MOE_TOPK_CASE
  return cudaErrorInvalidValue;
}

}  // namespace moe
