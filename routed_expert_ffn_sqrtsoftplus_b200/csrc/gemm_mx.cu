// Grouped expert GEMMs for block-scaled routed experts on tcgen05 block-scaled MMAs.
//
// Routed expert weights are MXFP4 (E2M1 values, one E8M0 scale per 32 along K;
// DeepSeek V4.1 config "expert_dtype": "fp4", MAX encoding float4_e2m1fnx2) or
// MXFP8 (E4M3 values, the same scales; MAX encoding float8_e4m3fn) and the
// activations they meet are MXFP8 (E4M3, one E8M0 scale per 32), so every MMA
// is tcgen05.mma.kind::mxf8f6f4.block_scale: A = 128 weight rows (E2M1, unpacked
// to one byte per value in shared memory by the 16U4_ALIGN16B TMA type, or E4M3
// loaded as it is stored), B = token rows (E4M3), scale factors in TMEM, fp32
// accumulation.
//
// Same persistent, warp-specialised structure as the BF16 kernel (warp 0 TMA,
// warp 1 MMA, 8 epilogue warps, two per TMEM lane quarter taking interleaved
// 16-column chunks; smem ring + two TMEM accumulators). One
// stage covers 128 values of K: A box 128 x (256 | 128) rows, B boxes 128 x 32
// token rows, and two 1-D bulk copies of pre-arranged scale-factor atoms (512 B
// per 128 rows x 4 blocks of 32). The MMA warp copies the atoms into this
// stage's TMEM scale columns with tcgen05.cp and issues four K=32 MMAs per
// matrix, selecting the block inside the atom with the scale-factor id.
//
//   gate/up: h = silu(min(G, L)) * clamp(U, -L, L), quantised to MXFP8 along the
//            expert width (a warp owns 32 consecutive rows of I, so the block
//            amax is a warp reduction) -> E4M3 rows + scale atoms for the down GEMM
//   down:    fp32 rows, as in the BF16 path; with kWide a tile covers 256 rows
//            of W2 (two MMAs sharing the token box, twice the HBM bytes per
//            ring stage)
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kEpiWarps = 8;  // two per TMEM lane quarter
constexpr int kEpiGroups = kEpiWarps / 4;
// Packed staging of MXFP4 weights (MOE_MX_PACKED, kernels.h): the ring holds the
// packed E2M1 bytes as stored (half the shared memory per HBM byte of the TMA
// unpacking), and kExpWarps expander warps copy each stage into the 16-byte-
// aligned layout the MMA reads, in kXBufs buffers of their own.
constexpr int kExpWarps = kMxPacked ? 4 : 0;
constexpr int kXBufs = MOE_MX_PACKED_BUFS;
static_assert(kXBufs == 1 || kXBufs == 2, "expanded buffers");
constexpr int kThreads = 64 + 32 * (kEpiWarps + kExpWarps);
constexpr int kBK = 128;          // K values per stage
constexpr int kBBoxRows = 32;
constexpr int kBBoxBytes = kBBoxRows * 128;
constexpr int kAtomBytes = 512;   // scale factors of 128 rows x 4 blocks
// Weight boxes prefetched into L2 this many ring stages ahead of the loads (0 = none).
#ifndef MOE_MX_PREFETCH
#define MOE_MX_PREFETCH 0
#endif
constexpr int kPrefetch = MOE_MX_PREFETCH;
// At the start of each tile, prefetch into L2 this many quarters of the weights
// of the CTA's next tile (contiguous in the repacked layout) with bulk prefetches
// (0 = none).
#ifndef MOE_MX_TILE_PREFETCH
#define MOE_MX_TILE_PREFETCH 0
#endif
constexpr int kTilePrefetchQuarters = MOE_MX_TILE_PREFETCH;

constexpr int pow2_at_least(int v, int lo) {
  int p = lo;
  while (p < v) p *= 2;
  return p;
}

// kWide (down GEMM): a tile covers 256 rows of W2, two 128-row MMAs sharing the
// token tile, like the gate/up tile's W1 and W3 halves.
// kAF8: A (the weights) is E4M3, one byte per value in HBM and in shared memory;
// otherwise E2M1, packed two per byte in HBM and unpacked to one per byte by the TMA.
template <bool kGateUp, bool kWide, int BN, int kStages, bool kAF8>
struct MxCfg {
  static constexpr bool kTwoA = kGateUp || kWide;       // two 128-row MMAs per K step
  static constexpr int kARows = kTwoA ? 256 : 128;
  static constexpr int kABytes = kARows * 128;          // one byte per value in shared memory
  static constexpr int kATx = kAF8 ? kABytes : kARows * 64;  // bytes the TMA moves from HBM
  static constexpr bool kPack = kMxPacked && !kAF8;     // packed staging (E2M1 only)
  static constexpr int kStageABytes = kPack ? kATx : kABytes;  // A bytes of one ring stage
  static constexpr int kNX = kPack ? kXBufs : 0;        // expanded A buffers
  static constexpr int kBBytes = BN * 128;
  static constexpr int kSfaBytes = kTwoA ? 2 * kAtomBytes : kAtomBytes;
  static constexpr int kSfBytes = kSfaBytes + kAtomBytes;
  static constexpr int kAccCols = kTwoA ? 2 * BN : BN;
  static constexpr int kSfCols = kTwoA ? 12 : 8;         // 4 TMEM columns per atom
  static constexpr int kSfColBase = 2 * kAccCols;
  static constexpr int kTmemCols = pow2_at_least(kSfColBase + kStages * kSfCols, 32);
  static constexpr int kBarrierBytes = 512;
  static constexpr int kSmemBytes =
      1024 + kNX * kABytes + kStages * (kStageABytes + kBBytes + kSfBytes) + kBarrierBytes;
  static_assert(kTmemCols <= 512, "TMEM");
  static_assert((2 * kStages + 5 + 2 * kNX) * 8 + 8 <= kBarrierBytes, "barriers");
  static_assert(BN % kBBoxRows == 0 && BN <= 128, "BN");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

struct Tile {
  int group, m_tile, ntile, row0, nrows;
};

template <int BN>
__device__ __forceinline__ Tile load_tile(const MxGemmArgs& a, int t) {
  const int4 v = a.tiles[t];
  Tile r;
  r.group = v.x & 0xFFFF;
  r.m_tile = v.x >> 16;
  r.ntile = v.y;
  r.row0 = v.z;
  r.nrows = max(0, min(v.w, BN));
  return r;
}

__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, const MxGemmArgs& a,
                                              volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > a.timeout_ns) {
      *abort_flag = 1;
      report_status(a.status, kStatusTimeout);
      return false;
    }
  }
}

template <bool kGateUp, bool kWide, int BN, int kStages, bool kAF8>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_mx_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                           const MxGemmArgs args) {
  using C = MxCfg<kGateUp, kWide, BN, kStages, kAF8>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sX = smem;                                   // expanded A buffers (packed staging)
  uint8_t* sA = sX + C::kNX * C::kABytes;
  uint8_t* sB = sA + kStages * C::kStageABytes;
  uint8_t* sSF = sB + kStages * C::kBBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sSF + kStages * C::kSfBytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + kStages;
  uint64_t* tfull = bars + 2 * kStages;
  uint64_t* tempty = bars + 2 * kStages + 2;
  uint64_t* drain = bars + 2 * kStages + 4;
  uint64_t* xfull = bars + 2 * kStages + 5;             // expanded buffer written
  uint64_t* xempty = xfull + C::kNX;                    // expanded buffer consumed by the MMAs
  uint32_t* tmem_base_smem = reinterpret_cast<uint32_t*>(xempty + C::kNX);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_smem + 1);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], kEpiWarps);
    }
    mbar_init(drain, 1);
    for (int i = 0; i < C::kNX; ++i) {
      mbar_init(&xfull[i], kExpWarps);
      mbar_init(&xempty[i], 1);
    }
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_base_smem, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_base_smem;

  const int tend = *args.ntiles;
  const int tfirst = (args.tile_begin ? *args.tile_begin : 0) + static_cast<int>(blockIdx.x);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      long issued = 0;
      // L2 prefetch cursor: walks the same (tile, K block) sequence kPrefetch stages ahead
      int pf_t = tfirst, pf_kb = 0, pf_row = 0;
      auto prefetch_next = [&]() {
        if (pf_t >= tend) return;
        if (pf_kb == 0) {
          const Tile pt = load_tile<BN>(args, pf_t);
          pf_row = pt.group * args.a_rows_per_group + pt.m_tile * C::kARows;
        }
        tma_prefetch_2d(&tmA, pf_kb * kBK, pf_row);
        if (++pf_kb == args.num_kb) {
          pf_kb = 0;
          pf_t += gridDim.x;
        }
      };
      if constexpr (kPrefetch > 0)
        for (int i = 0; i < kPrefetch; ++i) prefetch_next();
      for (int t = tfirst; t < tend && !*abort_flag; t += gridDim.x) {
        const Tile tl = load_tile<BN>(args, t);
        const int a_row = tl.group * args.a_rows_per_group + tl.m_tile * C::kARows;
        if constexpr (kTilePrefetchQuarters > 0) {
          if (t + static_cast<int>(gridDim.x) < tend && args.a_base != nullptr) {
            const Tile nt = load_tile<BN>(args, t + gridDim.x);
            const uint8_t* src = args.a_base + (static_cast<size_t>(nt.group) * args.a_rows_per_group +
                                                static_cast<size_t>(nt.m_tile) * C::kARows) * args.a_row_bytes;
            const size_t total = static_cast<size_t>(C::kARows) * args.a_row_bytes * kTilePrefetchQuarters / 4;
            for (size_t o = 0; o + 32768 <= total; o += 32768) bulk_prefetch_l2(src + o, 32768);
          }
        }
        const int nb = (tl.nrows + kBBoxRows - 1) / kBBoxRows;
        const uint32_t bytes = C::kATx + nb * kBBoxBytes + C::kSfBytes;
        // W1|W3 atoms: [group][m tile][k block][2 x 512 B]; W2 atoms: [group][128-row
        // tile][k block][512 B] (a wide tile takes 128-row tiles 2m and 2m + 1)
        const uint8_t* sfa_src =
            kWide ? args.sfa + (static_cast<size_t>(tl.group) * args.m_tiles + 2 * tl.m_tile) * args.num_kb * kAtomBytes
                  : args.sfa + (static_cast<size_t>(tl.group) * args.m_tiles + tl.m_tile) * args.num_kb * C::kSfaBytes;
        const uint8_t* sfb_src = args.sfb + static_cast<size_t>(tl.ntile) * args.num_kb * kAtomBytes;
        bool ok = true;
        for (int kb = 0; kb < args.num_kb; ++kb) {
          if (!wait_or_abort(&empty[stage], phase ^ 1, args, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], bytes);
          // packed staging: the A map is over bytes (kBK / 2 per K step); otherwise over values
          tma_load_2d(sA + stage * C::kStageABytes, &tmA, &full[stage], C::kPack ? kb * (kBK / 2) : kb * kBK, a_row,
                      kCacheEvictFirst);
          for (int j = 0; j < nb; ++j)
            tma_load_2d(sB + stage * C::kBBytes + j * kBBoxBytes, &tmB, &full[stage], kb * kBK,
                        tl.row0 + j * kBBoxRows, kCacheEvictLast);
          uint8_t* sf = sSF + stage * C::kSfBytes;
          if (kWide) {
            bulk_load(sf, sfa_src + static_cast<size_t>(kb) * kAtomBytes, kAtomBytes, &full[stage], kCacheEvictFirst);
            bulk_load(sf + kAtomBytes, sfa_src + static_cast<size_t>(args.num_kb + kb) * kAtomBytes, kAtomBytes,
                      &full[stage], kCacheEvictFirst);
          } else {
            bulk_load(sf, sfa_src + static_cast<size_t>(kb) * C::kSfaBytes, C::kSfaBytes, &full[stage],
                      kCacheEvictFirst);
          }
          bulk_load(sf + C::kSfaBytes, sfb_src + static_cast<size_t>(kb) * kAtomBytes, kAtomBytes, &full[stage],
                    kCacheEvictLast);
          if constexpr (kPrefetch > 0) prefetch_next();
          ++issued;
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
      }
      if (*abort_flag) {
        for (long i = issued - 1; i >= 0 && i >= issued - kStages; --i) {
          const int s = static_cast<int>(i % kStages);
          const uint32_t par = static_cast<uint32_t>((i / kStages) & 1);
          const uint64_t t0 = globaltimer_ns();
          while (!mbar_try_wait(&full[s], par) && globaltimer_ns() - t0 < args.timeout_ns) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      int xb = 0;
      uint32_t xph = 0;
      for (int t = tfirst; t < tend && !*abort_flag; t += gridDim.x) {
        const Tile tl = load_tile<BN>(args, t);
        const uint32_t n_mma = max(16, (tl.nrows + 15) & ~15);
        if (!wait_or_abort(&tempty[acc], acc_phase ^ 1, args, abort_flag)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + acc * C::kAccCols;
        bool ok = true;
        for (int kb = 0; kb < args.num_kb; ++kb) {
          if (!wait_or_abort(&full[stage], phase, args, abort_flag) ||
              (C::kPack && !wait_or_abort(&xfull[xb], xph, args, abort_flag))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = C::kPack ? smem_u32(sX + xb * C::kABytes) : smem_u32(sA + stage * C::kABytes);
          const uint32_t b_addr = smem_u32(sB + stage * C::kBBytes);
          const uint32_t sf_addr = smem_u32(sSF + stage * C::kSfBytes);
          const uint32_t sf_cols = tmem_base + C::kSfColBase + stage * C::kSfCols;
          // scale factors of this stage -> TMEM (replicated to all four lane quarters)
          tmem_cp_32x128b_x4(sf_cols, sdesc_plain(sf_addr));
          if (C::kTwoA) tmem_cp_32x128b_x4(sf_cols + 4, sdesc_plain(sf_addr + kAtomBytes));
          const uint32_t sfb_col = sf_cols + (C::kTwoA ? 8 : 4);
          tmem_cp_32x128b_x4(sfb_col, sdesc_plain(sf_addr + C::kSfaBytes));
#pragma unroll
          for (uint32_t k = 0; k < kBK / 32; ++k) {
            const uint32_t idesc = kAF8 ? idesc_mx_e4m3_e4m3(128, n_mma, k, k) : idesc_mx_e2m1_e4m3(128, n_mma, k, k);
            const uint64_t bdesc = sdesc_sw128(b_addr + k * 32);
            const uint32_t accum = (kb | k) != 0;
            umma_mx(d, sdesc_sw128(a_addr + k * 32), bdesc, idesc, sf_cols | (k << 30), sfb_col | (k << 30),
                    accum);
            if (C::kTwoA)
              umma_mx(d + BN, sdesc_sw128(a_addr + 128 * 128 + k * 32), bdesc, idesc, (sf_cols + 4) | (k << 30),
                      sfb_col | (k << 30), accum);
          }
          umma_commit(&empty[stage]);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
          if constexpr (C::kPack) {
            umma_commit(&xempty[xb]);
            if (++xb == C::kNX) {
              xb = 0;
              xph ^= 1;
            }
          }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
      umma_commit(drain);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(drain, 0) && globaltimer_ns() - t0 < args.timeout_ns) {
      }
    }
  } else if (warp >= 2 + kEpiWarps) {
    // ------------------------------------------------------------ expanders (packed staging)
    // Each stage's packed A rows (64 bytes = 128 E2M1 values) become the layout the
    // 16U4_ALIGN16B TMA would have written: 8 packed bytes at the start of each
    // 16-byte chunk, chunk c of row r at position c ^ (r % 8) of the row's 128
    // bytes (128-byte swizzle, 8-row atoms of 1024 bytes).
    if constexpr (C::kPack) {
      const int et = (warp - 2 - kEpiWarps) * 32 + lane;  // 0 .. 32 * kExpWarps - 1
      int stage = 0;
      uint32_t phase = 0;
      int xb = 0;
      uint32_t xph = 0;
      bool ok = true;
      for (int t = tfirst; ok && t < tend; t += gridDim.x) {
        for (int kb = 0; kb < args.num_kb; ++kb) {
          if (lane == 0)
            ok = wait_or_abort(&full[stage], phase, args, abort_flag) &&
                 wait_or_abort(&xempty[xb], xph ^ 1, args, abort_flag);
          ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
          if (!ok) break;
          const uint8_t* src = sA + stage * C::kStageABytes;
          uint8_t* dst = sX + xb * C::kABytes;
#pragma unroll 4
          for (int p = et; p < C::kARows * 4; p += 32 * kExpWarps) {
            const int r = p >> 2, q = p & 3;
            const uint4 v = *reinterpret_cast<const uint4*>(src + r * 64 + q * 16);
            uint8_t* row = dst + (r >> 3) * 1024 + (r & 7) * 128;
            *reinterpret_cast<uint2*>(row + (((2 * q) ^ (r & 7)) << 4)) = make_uint2(v.x, v.y);
            *reinterpret_cast<uint2*>(row + (((2 * q + 1) ^ (r & 7)) << 4)) = make_uint2(v.z, v.w);
          }
          fence_proxy_async_smem();  // the tensor core reads what these generic stores wrote
          __syncwarp();
          if (lane == 0) mbar_arrive(&xfull[xb]);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
          if (++xb == C::kNX) {
            xb = 0;
            xph ^= 1;
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                    // TMEM lane quarter this warp may access
    const int cfirst = ((warp - 2) / 4) * 16;  // this warp's first 16-column chunk
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = tfirst; t < tend; t += gridDim.x) {
      const Tile tl = load_tile<BN>(args, t);
      const int n_mma = max(16, (tl.nrows + 15) & ~15);
      bool ok = true;
      if (lane == 0) ok = wait_or_abort(&tfull[acc], acc_phase, args, abort_flag);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * C::kAccCols;
      const int m = tl.m_tile * (kWide ? 256 : 128) + q * 32 + lane;
      const bool rows_ok = tl.row0 >= 0 && tl.row0 + tl.nrows <= args.out_rows;
      if (!rows_ok && lane == 0 && q == 0) report_status(args.status, kStatusDevice);
      const bool m_ok = m < args.m_limit && rows_ok;
      int down_base_row = 0, down_ntile_base = 0;
      if constexpr (kGateUp) {
        // row index of this tile inside its expert group, and the group's first
        // down-GEMM token tile (for the scale atoms of h)
        down_base_row = tl.row0 - args.group_off[tl.group];
        down_ntile_base = args.dn_ntile_base[tl.group];
      }
      for (int c0 = cfirst; c0 < n_mma; c0 += 16 * kEpiGroups) {
        uint32_t g[16];
        tmem_ld16(tb + c0, g);
        if constexpr (kGateUp) {
          uint32_t u[16];
          tmem_ld16(tb + BN + c0, u);
          tmem_ld_wait();
          uint8_t* hq = static_cast<uint8_t*>(args.out);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int n = c0 + j;
            const float hv = clamped_swiglu_f32(__uint_as_float(g[j]), __uint_as_float(u[j]), args.limit);
            // MXFP8 block of 32 consecutive rows of I = this warp's 32 lanes
            float amax = fabsf(hv);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
            int code;
            float inv;
            mx_scale(amax, 8, code, inv);
            const __nv_fp8_storage_t qv = __nv_cvt_float_to_fp8(hv * inv, __NV_SATFINITE, __NV_E4M3);
            if (n < tl.nrows && m_ok) {
              hq[static_cast<size_t>(tl.row0 + n) * args.out_ld + m] = qv;
              if (lane == 0) {
                const int jr = down_base_row + n;
                const int nt = down_ntile_base + jr / args.bn_dn;
                const int nd = jr % args.bn_dn;
                args.sf_out[(static_cast<size_t>(nt) * args.sf_out_kb4 + tl.m_tile) * kAtomBytes + (nd % 32) * 16 +
                            (nd / 32) * 4 + q] = static_cast<uint8_t>(code);
              }
            }
          }
        } else {
          tmem_ld_wait();
          float* out = static_cast<float*>(args.out);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int n = c0 + j;
            if (n < tl.nrows && m_ok) out[static_cast<size_t>(tl.row0 + n) * args.out_ld + m] = __uint_as_float(g[j]);
          }
          if constexpr (kWide) {
            // the second 128 rows of W2 (output columns m + 128)
            uint32_t g2[16];
            tmem_ld16(tb + BN + c0, g2);
            tmem_ld_wait();
            const bool m2_ok = m + 128 < args.m_limit && rows_ok;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int n = c0 + j;
              if (n < tl.nrows && m2_ok)
                out[static_cast<size_t>(tl.row0 + n) * args.out_ld + m + 128] = __uint_as_float(g2[j]);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

template <bool kGateUp, bool kWide, int BN, int kStages, bool kAF8>
cudaError_t set_attr() {
  return cudaFuncSetAttribute(grouped_gemm_mx_kernel<kGateUp, kWide, BN, kStages, kAF8>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              MxCfg<kGateUp, kWide, BN, kStages, kAF8>::kSmemBytes);
}

template <bool kGateUp, bool kWide, int BN, int kStages, bool kAF8>
cudaError_t launch(const CUtensorMap& tmA, const CUtensorMap& tmB, const MxGemmArgs& a, int grid, cudaStream_t s) {
  grouped_gemm_mx_kernel<kGateUp, kWide, BN, kStages, kAF8>
      <<<grid, kThreads, MxCfg<kGateUp, kWide, BN, kStages, kAF8>::kSmemBytes, s>>>(tmA, tmB, a);
  return cudaGetLastError();
}

// Ring depths: as many stages as fit in 227 KB.
constexpr int mx_ring_fit(int a_bytes, int b_bytes, int sf_bytes, int fixed) {
  return (227 * 1024 - 1024 - 512 - fixed) / (a_bytes + b_bytes + sf_bytes);
}
// Ring stages for a token-tile width, one or two 128-row weight MMAs, packed staging or not:
//   unpacked  two A: 32: 6, 64: 5, 96: 4    one A: 32: 10, 64: 9, 96: 7
//   packed    two A (2 expanded buffers): 32: 7, 64: 6, 96: 5
template <int BN, bool kTwo, bool kPack>
constexpr int kStagesFor =
    kPack ? mx_ring_fit((kTwo ? 256 : 128) * 64, BN * 128, (kTwo ? 3 : 2) * kAtomBytes, kXBufs * (kTwo ? 256 : 128) * 128)
          : mx_ring_fit((kTwo ? 256 : 128) * 128, BN * 128, (kTwo ? 3 : 2) * kAtomBytes, 0);
constexpr bool kExtraWidth = kBnMxLarge != 32 && kBnMxLarge != 64;

template <bool kGateUp, bool kWide, bool kAF8>
cudaError_t set_attrs() {
  constexpr bool two = kGateUp || kWide;
  cudaError_t e;
  if ((e = set_attr<kGateUp, kWide, 32, kStagesFor<32, two, kMxPacked && !kAF8>, kAF8>()) != cudaSuccess) return e;
  if ((e = set_attr<kGateUp, kWide, 64, kStagesFor<64, two, kMxPacked && !kAF8>, kAF8>()) != cudaSuccess) return e;
  if constexpr (kExtraWidth)
    if ((e = set_attr<kGateUp, kWide, kBnMxLarge, kStagesFor<kBnMxLarge, two, kMxPacked && !kAF8>,
                      kAF8>()) != cudaSuccess)
      return e;
  return cudaSuccess;
}

template <bool kGateUp, bool kWide, bool kAF8>
cudaError_t launch_any(const CUtensorMap& tmA, const CUtensorMap& tmB, const MxGemmArgs& a, int bn, int grid,
                       cudaStream_t s) {
  constexpr bool two = kGateUp || kWide;
  if (bn == 32)
    return launch<kGateUp, kWide, 32, kStagesFor<32, two, kMxPacked && !kAF8>, kAF8>(tmA, tmB, a, grid, s);
  if (bn == 64)
    return launch<kGateUp, kWide, 64, kStagesFor<64, two, kMxPacked && !kAF8>, kAF8>(tmA, tmB, a, grid, s);
  if constexpr (kExtraWidth)
    if (bn == kBnMxLarge)
      return launch<kGateUp, kWide, kBnMxLarge, kStagesFor<kBnMxLarge, two, kMxPacked && !kAF8>, kAF8>(
          tmA, tmB, a, grid, s);
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t gemm_mx_set_attributes() {
  cudaError_t e;
  if ((e = set_attrs<true, false, false>()) != cudaSuccess) return e;
  if ((e = set_attrs<false, false, false>()) != cudaSuccess) return e;
  if ((e = set_attrs<false, true, false>()) != cudaSuccess) return e;
  if ((e = set_attrs<true, false, true>()) != cudaSuccess) return e;
  if ((e = set_attrs<false, false, true>()) != cudaSuccess) return e;
  if ((e = set_attrs<false, true, true>()) != cudaSuccess) return e;
  return cudaSuccess;
}

cudaError_t launch_gemm_mx_gateup(const CUtensorMap& tmA, const CUtensorMap& tmB, const MxGemmArgs& a, int bn,
                                  int grid, cudaStream_t s, bool a_fp8) {
  return a_fp8 ? launch_any<true, false, true>(tmA, tmB, a, bn, grid, s)
               : launch_any<true, false, false>(tmA, tmB, a, bn, grid, s);
}

cudaError_t launch_gemm_mx_down(const CUtensorMap& tmA, const CUtensorMap& tmB, const MxGemmArgs& a, int bn,
                                int grid, cudaStream_t s, bool wide, bool a_fp8) {
  if (a_fp8)
    return wide ? launch_any<false, true, true>(tmA, tmB, a, bn, grid, s)
                : launch_any<false, false, true>(tmA, tmB, a, bn, grid, s);
  return wide ? launch_any<false, true, false>(tmA, tmB, a, bn, grid, s)
              : launch_any<false, false, false>(tmA, tmB, a, bn, grid, s);
}

}  // namespace moe
