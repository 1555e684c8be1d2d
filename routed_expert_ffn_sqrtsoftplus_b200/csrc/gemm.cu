// Grouped expert GEMMs on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// Swap-AB formulation: the expert weights are the M operand (128 rows of the
// weight matrix per MMA) and the tokens routed to the expert are the N operand
// (16..BN tokens), so a decode step with 1-3 tokens per expert still issues
// full-height MMAs while streaming every weight byte exactly once.
//
//   gate/up tile: D_G[128 x N] = W1[rows] . X^T,  D_U[128 x N] = W3[rows] . X^T
//                 h[token, i] = silu(min(D_G, L)) * clamp(D_U, -L, L)   -> BF16
//                 (the gated expert MLP with the swiglu_limit clamp of the
//                 DeepSeek V4.1 config: "swiglu_limit": 10.0)
//   down tile:    D[128 x N] = W2[rows] . h^T (one or two 128-row MMAs) -> fp32 rows
//
// One persistent CTA per SM, warp-specialised:
//   warp 0      TMA producer: per 64-wide K step one A box (weights) and the B
//               boxes (token rows) into one stage of the shared-memory ring
//   warp 1      MMA issuer: tcgen05.mma kind::f16, accumulators in TMEM
//   warps 2..   epilogue (kEpiWarps): tcgen05.ld -> math -> global stores; warp w
//               reads TMEM lane quarter w % 4, and the kEpiWarps / 4 warps of a
//               quarter take interleaved 16-column chunks of the tile
// A ring of full/empty mbarriers decouples TMA and MMA (weights and tokens of a
// stage travel together: separate, differently deep rings for the two measured
// slower on B200). One or two TMEM accumulator buffers (tmem_full/tmem_empty)
// let the epilogue of tile i overlap the MMAs of tile i+1 when they fit.
// grouped_gemm_dual_kernel holds two token-tile widths (two ring configurations)
// and runs the one the permutation kernel chose for this batch.
// Every wait is bounded in time; a wait that runs out records MOE_ERR_TIMEOUT,
// drains this CTA's in-flight copies and MMAs, frees TMEM and returns.
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

// 12: three warps per TMEM lane quarter. With one accumulator (256-token tiles) the
// MMAs wait for the epilogue, whose SwiGLU is latency-bound with two warps per
// scheduler; a third shortens it (V4-Pro gate/up 1.24 / 1.25 ms against 1.26 /
// 1.28 with 8 warps; 16 warps no better).
#ifndef MOE_EPI_WARPS
#define MOE_EPI_WARPS 12
#endif
constexpr int kEpiWarps = MOE_EPI_WARPS;  // a multiple of 4
// Epilogue rows staged in shared memory for 16-byte global stores where the ring
// leaves room (1), or stored one element per lane (0). Measured on V4-Pro: the
// gate/up's BF16 h rows gain (gate/up 1.25-1.27 ms against 1.27-1.29), the down's
// fp32 O rows lose (0.69-0.70 against 0.67-0.68), so only the former by default.
#ifndef MOE_EPI_STAGE
#define MOE_EPI_STAGE 1
#endif
#ifndef MOE_EPI_STAGE_DOWN
#define MOE_EPI_STAGE_DOWN 0
#endif
constexpr bool kEpiStage = MOE_EPI_STAGE != 0;
constexpr bool kEpiStageDown = MOE_EPI_STAGE_DOWN != 0;
constexpr int kEpiGroups = kEpiWarps / 4;
constexpr int kThreads = 64 + 32 * kEpiWarps;
static_assert(kEpiWarps % 4 == 0 && kEpiWarps >= 4 && kEpiWarps <= 16, "epilogue warps");
constexpr int kBK = 64;           // K elements per stage (128 bytes of BF16 = one swizzle row)
constexpr int kBBoxRows = 32;     // token rows per B TMA box
constexpr int kBBoxBytes = kBBoxRows * 128;
constexpr int kWarpTma = 0, kWarpMma = 1;
// Weight boxes prefetched into L2 this many ring stages ahead of the loads (0 = none).
#ifndef MOE_BF16_PREFETCH
#define MOE_BF16_PREFETCH 0
#endif
constexpr int kPrefetch = MOE_BF16_PREFETCH;

constexpr int pow2_at_least(int v, int lo) {
  int p = lo;
  while (p < v) p *= 2;
  return p;
}

// kAMmas 128-row MMAs per K step share one B tile: gate/up always has two (W1
// and W3 rows of the same 128 expert-width rows); the down GEMM has one, or two
// consecutive 128-row tiles of W2 ("wide") to double the work per B byte.
// Tile indices in flight from the producer to the MMA thread and the epilogue
// warps when the tiles come from a counter.
constexpr int kTileQ = 4;

template <bool kGateUp, int kAMmas, int BN, int kStages>
struct Cfg {
  static constexpr int kARows = 128 * kAMmas;
  static constexpr int kABytes = kARows * 128;
  static constexpr int kBBytes = BN * 128;
  static constexpr int kAccCols = kAMmas * BN;
  // two accumulator buffers when they fit in TMEM, otherwise one
  static constexpr int kAccBufs = 2 * kAccCols <= 512 ? 2 : 1;
  static constexpr int kTmemCols = pow2_at_least(kAccBufs * kAccCols, 32);
  static constexpr int kBarrierBytes = 512;
  static constexpr int kBaseBytes = 1024 + kStages * (kABytes + kBBytes) + kBarrierBytes;
  // Epilogue staging, when it fits beside the ring: each epilogue warp turns its 16 x 32
  // chunk into 16-byte row segments for the global stores (kEpiStage: BF16 h rows of
  // the gate/up GEMM; fp32 O rows with kEpiStageDown).
  static constexpr int kStageWarpBytes = kGateUp ? 16 * 32 * 2 : 16 * 32 * 4;
  static constexpr bool kStaged = kGateUp ? kEpiStage : kEpiStageDown;
  static constexpr int kStageBytes =
      kStaged && kBaseBytes + kEpiWarps * kStageWarpBytes <= 227 * 1024 ? kEpiWarps * kStageWarpBytes : 0;
  static constexpr int kSmemBytes = kBaseBytes + kStageBytes;
  static_assert(!kGateUp || kAMmas == 2, "gate/up tiles pair W1 and W3 rows");
  static_assert(kTmemCols <= 512, "TMEM holds 512 columns");
  static_assert(BN % kBBoxRows == 0 && BN >= 32 && BN <= 256, "BN");
  static_assert((2 * kStages + 5 + 2 * kTileQ) * 8 + 8 + 4 * kTileQ <= kBarrierBytes, "barriers");
  static_assert(kSmemBytes <= 227 * 1024, "shared memory");
};

struct Tile {
  int group, m_tile, b_row0, out_row0, nrows;
  int kb0, nkb, split;  // K blocks [kb0, kb0 + nkb) of slice `split`
};

template <int BN>
__device__ __forceinline__ Tile load_tile(const GemmArgs& a, int t) {
  Tile r;
  r.kb0 = 0;
  r.nkb = a.num_kb;
  r.split = 0;
  if (a.tiles != nullptr) {
    const int4 v = a.tiles[t];
    r.group = v.x & 0xFFFF;
    r.m_tile = v.x >> 16;
    r.b_row0 = v.y;
    r.out_row0 = v.z;
    r.nrows = v.w;
  } else {
    // dense: m fastest, then K slice, then token tile
    const int ks = max(1, a.dense_k_splits);
    r.group = 0;
    r.m_tile = t % a.dense_m_tiles;
    const int rest = t / a.dense_m_tiles;
    r.split = rest % ks;
    const int nt = rest / ks;
    r.nkb = a.num_kb / ks;
    r.kb0 = r.split * r.nkb;
    r.out_row0 = nt * BN;
    r.b_row0 = a.dense_b_row0 + nt * BN;
    r.nrows = min(BN, a.dense_rows - nt * BN);
  }
  // A tile never holds more rows than the B ring has room for.
  r.nrows = max(0, min(r.nrows, BN));
  return r;
}

template <int BN>
__device__ __forceinline__ int tile_count(const GemmArgs& a) {
  if (a.tiles != nullptr) return *a.ntiles;
  return a.dense_m_tiles * max(1, a.dense_k_splits) * ((a.dense_rows + BN - 1) / BN);
}

__device__ __forceinline__ int tile_first(const GemmArgs& a) {
  return (a.tiles != nullptr && a.tile_begin != nullptr) ? *a.tile_begin : 0;
}

// Wait that also gives up as soon as another role of this CTA has aborted.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, const GemmArgs& a,
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

// After an abort: wait (bounded) until the last `depth` copies this thread
// issued into a ring have landed, so no copy writes into a CTA that is gone.
__device__ __forceinline__ void drain_ring(uint64_t* full, int depth, long issued, uint64_t timeout_ns) {
  for (long i = issued - 1; i >= 0 && i >= issued - depth; --i) {
    const int s = static_cast<int>(i % depth);
    const uint32_t par = static_cast<uint32_t>((i / depth) & 1);
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(&full[s], par) && globaltimer_ns() - t0 < timeout_ns) {
    }
  }
}

// Before the ring's shared memory is reused: wait (bounded) until the MMAs have
// released every stage, so no commit still has to arrive on an empty barrier.
template <int kStages>
__device__ __forceinline__ void release_ring(uint64_t* empty, int stage, uint32_t phase, const GemmArgs& a,
                                             volatile int* abort_flag) {
  for (int i = 0; i < kStages; ++i) {
    if (!wait_or_abort(&empty[stage], phase ^ 1, a, abort_flag)) return;
    if (++stage == kStages) {
      stage = 0;
      phase ^= 1;
    }
  }
}

// Runs tiles [tlo, thi) of the list: every gridDim-th from tlo + blockIdx.x, or,
// with `counter`, tlo + the counter's next value until that reaches thi (the
// producer takes the index and hands it to the MMA thread and the epilogue warps
// through a small queue in shared memory). With `again` another body follows in
// the same CTA: TMEM is freed without giving up the right to allocate it, and the
// barriers are invalidated so that their shared memory can be reused. Returns
// false when the CTA aborted (timeout).
template <bool kGateUp, int kAMmas, int BN, int kStages>
__device__ __forceinline__ bool gemm_body(const CUtensorMap* tmA, const CUtensorMap* tmB, const CUtensorMap* tmBsh,
                                          const GemmArgs& args, uint8_t* smem_raw, int tlo, int thi,
                                          int* counter = nullptr, bool again = false) {
  using C = Cfg<kGateUp, kAMmas, BN, kStages>;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kStages * C::kABytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + kStages * C::kBBytes);
  uint64_t* full = bars;
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* tq_full = drain + 1;       // tile queue: index written
  uint64_t* tq_empty = tq_full + kTileQ;  // tile queue: index read by the MMA thread and every epilogue warp
  constexpr int kNumBars = 2 * kStages + 5 + 2 * kTileQ;
  uint32_t* tmem_base_smem = reinterpret_cast<uint32_t*>(tq_empty + kTileQ);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_smem + 1);
  volatile int* tq = reinterpret_cast<volatile int*>(tmem_base_smem + 2);
  uint8_t* stage_base = reinterpret_cast<uint8_t*>(bars) + C::kBarrierBytes;  // C::kStageBytes of staging

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], kEpiWarps);  // one arrive per epilogue warp
    }
    mbar_init(drain, 1);
    for (int i = 0; i < kTileQ; ++i) {
      mbar_init(&tq_full[i], 1);
      mbar_init(&tq_empty[i], 1 + kEpiWarps);
    }
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == kWarpTma && lane == 0) {
    tma_prefetch_desc(tmA);
    tma_prefetch_desc(tmB);
    if (kGateUp) tma_prefetch_desc(tmBsh);
  }
  if (warp == kWarpMma) {
    tmem_alloc(tmem_base_smem, C::kTmemCols);
    if (!again) tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_base_smem;

  const int ntiles = thi;
  const int tfirst = tlo + static_cast<int>(blockIdx.x);
  const bool dyn = counter != nullptr;
  // the tile after `prev` (-1: the first), or -1 when there is none
  auto stride_next = [&](int prev) -> int {
    const int t = prev < 0 ? tfirst : prev + static_cast<int>(gridDim.x);
    return t < ntiles ? t : -1;
  };
  // producer (one thread): next tile, published to the queue when dynamic
  int tq_ps = 0;
  uint32_t tq_pp = 0;
  auto produce = [&](int prev) -> int {
    if (!dyn) return stride_next(prev);
    int t = tlo + atomicAdd(counter, 1);
    if (t >= ntiles) t = -1;
    if (!wait_or_abort(&tq_empty[tq_ps], tq_pp ^ 1, args, abort_flag)) return -1;
    tq[tq_ps] = t;
    mbar_arrive(&tq_full[tq_ps]);
    if (++tq_ps == kTileQ) {
      tq_ps = 0;
      tq_pp ^= 1;
    }
    return t;
  };
  // consumers (the MMA thread, lane 0 of each epilogue warp): the producer's sequence
  int tq_cs = 0;
  uint32_t tq_cp = 0;
  auto consume = [&](int prev) -> int {
    if (!dyn) return stride_next(prev);
    if (!wait_or_abort(&tq_full[tq_cs], tq_cp, args, abort_flag)) return -1;
    const int t = tq[tq_cs];
    mbar_arrive(&tq_empty[tq_cs]);
    if (++tq_cs == kTileQ) {
      tq_cs = 0;
      tq_cp ^= 1;
    }
    return t;
  };

  if (warp == kWarpTma) {
    // ------------------------------------------------------------ TMA producer
    if constexpr (!kGatherX) {
      // lane 0 waits on the ring and issues the weight box and the token boxes
      if (lane == 0) {
        int stage = 0;
        uint32_t phase = 0;
        long issued = 0;
        bool ok = true;
        // L2 prefetch cursor: walks the same (tile, K block) sequence kPrefetch stages ahead
        int pf_t = tfirst, pf_kb = 0, pf_row = 0, pf_kb0 = 0, pf_nkb = 0;
        auto prefetch_next = [&]() {
          if (pf_t >= ntiles) return;
          if (pf_kb == 0) {
            const Tile pt = load_tile<BN>(args, pf_t);
            pf_row = (pt.group - args.group_base) * args.a_rows_per_group + pt.m_tile * C::kARows;
            pf_kb0 = pt.kb0;
            pf_nkb = pt.nkb;
          }
          if (pf_nkb > 0) tma_prefetch_2d(tmA, (pf_kb0 + pf_kb) * kBK, pf_row);
          if (++pf_kb >= pf_nkb) {
            pf_kb = 0;
            pf_t += gridDim.x;
          }
        };
        if constexpr (kPrefetch > 0)
          if (!dyn)
            for (int i = 0; i < kPrefetch; ++i) prefetch_next();
        for (int t = produce(-1); ok && t >= 0 && !*abort_flag; t = produce(t)) {
          const Tile tl = load_tile<BN>(args, t);
          const CUtensorMap* mb = (kGateUp && tl.group >= args.n_routed) ? tmBsh : tmB;
          const int a_row = (tl.group - args.group_base) * args.a_rows_per_group + tl.m_tile * C::kARows;
          const int nb = (tl.nrows + kBBoxRows - 1) / kBBoxRows;
          const uint32_t bytes = C::kABytes + nb * kBBoxBytes;
          for (int kb = 0; kb < tl.nkb; ++kb) {
            if (!wait_or_abort(&empty[stage], phase ^ 1, args, abort_flag)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&full[stage], bytes);
            const int kx = (tl.kb0 + kb) * kBK;
            tma_load_2d(sA + stage * C::kABytes, tmA, &full[stage], kx, a_row, kCacheEvictFirst);
            for (int j = 0; j < nb; ++j)
              tma_load_2d(sB + stage * C::kBBytes + j * kBBoxBytes, mb, &full[stage], kx, tl.b_row0 + j * kBBoxRows,
                          kCacheEvictLast);
            if constexpr (kPrefetch > 0)
              if (!dyn) prefetch_next();
            ++issued;
            if (++stage == kStages) {
              stage = 0;
              phase ^= 1;
            }
          }
        }
        if (*abort_flag) drain_ring(full, kStages, issued, args.timeout_ns);
        else if (again) release_ring<kStages>(empty, stage, phase, args, abort_flag);
      }
    } else {
      // Lane 0 waits on the ring and issues the weight box (and the token boxes of
      // rows stored in order); with gathered token rows every lane issues the
      // tile::gather4 loads of its own four-row groups.
      constexpr int kGpl = (BN / 4 + 31) / 32;  // four-row groups per lane
      int stage = 0;
      uint32_t phase = 0;
      long issued = 0;
      bool ok = true;
      // L2 prefetch cursor (lane 0): walks the same (tile, K block) sequence kPrefetch stages ahead
      int pf_t = tfirst, pf_kb = 0, pf_row = 0, pf_kb0 = 0, pf_nkb = 0;
      auto prefetch_next = [&]() {
        if (pf_t >= ntiles) return;
        if (pf_kb == 0) {
          const Tile pt = load_tile<BN>(args, pf_t);
          pf_row = (pt.group - args.group_base) * args.a_rows_per_group + pt.m_tile * C::kARows;
          pf_kb0 = pt.kb0;
          pf_nkb = pt.nkb;
        }
        if (pf_nkb > 0) tma_prefetch_2d(tmA, (pf_kb0 + pf_kb) * kBK, pf_row);
        if (++pf_kb >= pf_nkb) {
          pf_kb = 0;
          pf_t += gridDim.x;
        }
      };
      if constexpr (kPrefetch > 0)
        if (lane == 0 && !dyn)
          for (int i = 0; i < kPrefetch; ++i) prefetch_next();
      for (int t = __shfl_sync(0xffffffffu, lane == 0 ? produce(-1) : 0, 0); ok && t >= 0;
           t = __shfl_sync(0xffffffffu, lane == 0 ? produce(t) : 0, 0)) {
        if (__shfl_sync(0xffffffffu, lane == 0 ? *abort_flag : 0, 0)) break;
        const Tile tl = load_tile<BN>(args, t);
        const bool gather = kGateUp && args.gather_perm != nullptr && tl.group < args.n_routed;
        const CUtensorMap* mb = (kGateUp && tl.group >= args.n_routed) ? tmBsh : tmB;
        const int a_row = (tl.group - args.group_base) * args.a_rows_per_group + tl.m_tile * C::kARows;
        const int nb = (tl.nrows + kBBoxRows - 1) / kBBoxRows;
        const int n4 = (tl.nrows + 3) / 4;
        // token rows of this lane's four-row groups (the tile's last row repeated past its end)
        int tok[kGpl][4];
  #pragma unroll
        for (int u = 0; u < kGpl; ++u)
  #pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int r = min(4 * (lane + 32 * u) + i, tl.nrows - 1);
            tok[u][i] = (gather && r >= 0) ? args.gather_perm[tl.b_row0 + r] / args.gather_k : 0;
          }
        const uint32_t bytes = C::kABytes + (gather ? n4 * 4 * 128 : nb * kBBoxBytes);
        for (int kb = 0; kb < tl.nkb; ++kb) {
          int go = 1;
          if (lane == 0) go = wait_or_abort(&empty[stage], phase ^ 1, args, abort_flag) ? 1 : 0;
          if (!__shfl_sync(0xffffffffu, go, 0)) {
            ok = false;
            break;
          }
          const int kx = (tl.kb0 + kb) * kBK;
          if (lane == 0) {
            mbar_arrive_expect_tx(&full[stage], bytes);
            tma_load_2d(sA + stage * C::kABytes, tmA, &full[stage], kx, a_row, kCacheEvictFirst);
            if (!gather)
              for (int j = 0; j < nb; ++j)
                tma_load_2d(sB + stage * C::kBBytes + j * kBBoxBytes, mb, &full[stage], kx, tl.b_row0 + j * kBBoxRows,
                            kCacheEvictLast);
            if constexpr (kPrefetch > 0)
              if (!dyn) prefetch_next();
          }
          __syncwarp();
          if (gather) {
  #pragma unroll
            for (int u = 0; u < kGpl; ++u) {
              const int g = lane + 32 * u;
              if (g < n4)
                tma_gather4(sB + stage * C::kBBytes + g * 4 * 128, tmB, &full[stage], kx, tok[u][0], tok[u][1],
                            tok[u][2], tok[u][3]);
            }
          }
          ++issued;
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (lane == 0 && *abort_flag) drain_ring(full, kStages, issued, args.timeout_ns);
      else if (lane == 0 && again) release_ring<kStages>(empty, stage, phase, args, abort_flag);
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = consume(-1); ok && t >= 0 && !*abort_flag; t = consume(t)) {
        const Tile tl = load_tile<BN>(args, t);
        const uint32_t n_mma = max(16, (tl.nrows + 15) & ~15);
        const uint32_t idesc = idesc_bf16_f32(128, n_mma);
        if (!wait_or_abort(&tempty[acc], acc_phase ^ 1, args, abort_flag)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + acc * C::kAccCols;
        for (int kb = 0; kb < tl.nkb; ++kb) {
          if (!wait_or_abort(&full[stage], phase, args, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * C::kABytes);
          const uint32_t b_addr = smem_u32(sB + stage * C::kBBytes);
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            const uint64_t bdesc = sdesc_sw128(b_addr + k * 32);
            const uint32_t accum = (kb | k) != 0;
#pragma unroll
            for (int i = 0; i < kAMmas; ++i)
              umma_f16(d + i * BN, sdesc_sw128(a_addr + i * 128 * 128 + k * 32), bdesc, idesc, accum);
          }
          umma_commit(&empty[stage]);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
        if (++acc == C::kAccBufs) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
      // Every MMA this thread issued has completed once `drain` flips.
      umma_commit(drain);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(drain, 0) && globaltimer_ns() - t0 < args.timeout_ns) {
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..)
    const int q = warp & 3;                  // TMEM lane quarter this warp may access
    const int cfirst = ((warp - 2) / 4) * 16;  // this warp's first 16-column chunk
    // 16-byte stores need rows and the output's column count a multiple of 8 elements
    const bool vec_out = args.out_ld % 8 == 0 && args.m_limit % 8 == 0;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = __shfl_sync(0xffffffffu, lane == 0 ? consume(-1) : 0, 0); t >= 0;
         t = __shfl_sync(0xffffffffu, lane == 0 ? consume(t) : 0, 0)) {
      const Tile tl = load_tile<BN>(args, t);
      const int n_mma = max(16, (tl.nrows + 15) & ~15);
      bool ok = true;
      if (lane == 0) ok = wait_or_abort(&tfull[acc], acc_phase, args, abort_flag);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * C::kAccCols;
      const int m = tl.m_tile * (kGateUp ? 128 : C::kARows) + q * 32 + lane;
      const bool rows_ok = tl.out_row0 >= 0 && tl.out_row0 + tl.nrows <= args.out_rows;
      if (!rows_ok && lane == 0 && q == 0) report_status(args.status, kStatusDevice);
      const bool m_ok = m < args.m_limit && rows_ok;
      for (int c0 = cfirst; c0 < n_mma; c0 += 16 * kEpiGroups) {
        uint32_t g[16];
        tmem_ld16(tb + c0, g);
        if constexpr (kGateUp) {
          uint32_t u[16];
          tmem_ld16(tb + BN + c0, u);
          tmem_ld_wait();
          if (args.raw_gateup) {
            // split-K partial sums: fp32 G at column m, U at column m_limit + m
            float* out = static_cast<float*>(args.out) + static_cast<size_t>(tl.split) * args.split_stride;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int n = c0 + j;
              if (n < tl.nrows && m_ok) {
                const size_t o = static_cast<size_t>(tl.out_row0 + n) * args.out_ld + m;
                out[o] = __uint_as_float(g[j]);
                out[o + args.m_limit] = __uint_as_float(u[j]);
              }
            }
          } else {
            __nv_bfloat16* out = static_cast<__nv_bfloat16*>(args.out);
            if (C::kStageBytes > 0 && vec_out) {
              // the warp's 16 token rows x 32 columns through shared memory, then 16-byte row segments
              __nv_bfloat16* sw = reinterpret_cast<__nv_bfloat16*>(stage_base) + (warp - 2) * 16 * 32;
#pragma unroll
              for (int j = 0; j < 16; ++j)
                sw[j * 32 + lane] =
                    __float2bfloat16_rn(clamped_swiglu_f32(__uint_as_float(g[j]), __uint_as_float(u[j]), args.limit));
              __syncwarp();
              const int mw = m - lane;  // the warp's first column
#pragma unroll
              for (int sg = lane; sg < 64; sg += 32) {
                const int r = sg >> 2, p = sg & 3, n = c0 + r;
                if (n < tl.nrows && rows_ok && mw + p * 8 + 8 <= args.m_limit)
                  *reinterpret_cast<uint4*>(out + static_cast<size_t>(tl.out_row0 + n) * args.out_ld + mw + p * 8) =
                      *reinterpret_cast<const uint4*>(sw + r * 32 + p * 8);
              }
              __syncwarp();
            } else {
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                const int n = c0 + j;
                if (n < tl.nrows && m_ok) {
                  const float hv = clamped_swiglu_f32(__uint_as_float(g[j]), __uint_as_float(u[j]), args.limit);
                  out[static_cast<size_t>(tl.out_row0 + n) * args.out_ld + m] = __float2bfloat16_rn(hv);
                }
              }
            }
          }
        } else {
          tmem_ld_wait();
          float* out = static_cast<float*>(args.out) + static_cast<size_t>(tl.split) * args.split_stride;
#pragma unroll
          for (int i = 0; i < kAMmas; ++i) {
            uint32_t v[16];
            if (i == 0) {
#pragma unroll
              for (int j = 0; j < 16; ++j) v[j] = g[j];
            } else {
              tmem_ld16(tb + i * BN + c0, v);
              tmem_ld_wait();
            }
            const int mi = m + i * 128;
            const bool ok_i = mi < args.m_limit && rows_ok;
            const float cb = (args.col_bias != nullptr && ok_i) ? args.col_bias[mi] : 0.0f;
            if (C::kStageBytes > 0 && vec_out) {
              // the warp's 16 rows x 32 columns through shared memory, then 16-byte row segments
              float* sw = reinterpret_cast<float*>(stage_base) + (warp - 2) * 16 * 32;
#pragma unroll
              for (int j = 0; j < 16; ++j) sw[j * 32 + lane] = __uint_as_float(v[j]) + cb;
              __syncwarp();
              const int mw = mi - lane;  // the warp's first column
#pragma unroll
              for (int sg = lane; sg < 128; sg += 32) {
                const int r = sg >> 3, p = sg & 7, n = c0 + r;
                if (n < tl.nrows && rows_ok && mw + p * 4 + 4 <= args.m_limit)
                  *reinterpret_cast<float4*>(out + static_cast<size_t>(tl.out_row0 + n) * args.out_ld + mw + p * 4) =
                      *reinterpret_cast<const float4*>(sw + r * 32 + p * 4);
              }
              __syncwarp();
            } else {
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                const int n = c0 + j;
                if (n < tl.nrows && ok_i)
                  out[static_cast<size_t>(tl.out_row0 + n) * args.out_ld + mi] = __uint_as_float(v[j]) + cb;
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (++acc == C::kAccBufs) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
  const bool ok = *abort_flag == 0;
  if (again) {
    // the next body's TMA copies may land where this body's epilogue staged rows
    fence_proxy_async_smem();
    __syncthreads();
    if (threadIdx.x == 0)
      for (int i = 0; i < kNumBars; ++i) mbar_inval(&bars[i]);
    __syncthreads();
  }
  return ok;
}

// Bounded wait until *p >= target (acquire); gives up when another role of the CTA
// has aborted or the time runs out (then records MOE_ERR_TIMEOUT and aborts).
__device__ __forceinline__ bool wait_count(const int* p, int target, const GemmArgs& a, volatile int* abort_flag) {
  if (ld_acquire_gpu(p) >= target) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i) {
      if (ld_acquire_gpu(p) >= target) return true;
      __nanosleep(100);
    }
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > a.timeout_ns) {
      *abort_flag = 1;
      report_status(a.status, kStatusTimeout);
      return false;
    }
  }
}

// Gate/up and down of the few-token path in one persistent launch. Both halves
// have the same geometry: two 128-row MMAs per K step sharing a BN-token tile (W1
// and W3 rows of 128 expert-width rows; two 128-row halves of 256 W2 rows), so one
// ring and one TMEM layout serve both. The combined tile index walks every gate/up
// tile and then every down tile; a CTA takes every gridDim-th one, so it has
// finished all its gate/up tiles before any down tile. A down tile of group g
// waits until all of g's gate/up tiles have stored h: each epilogue warp of such a
// tile adds 1 to done[g] after its stores, and g is ready at
// m_tiles_gu * token tiles * kEpiWarps. All CTAs are resident (cooperative
// launch), so every gate/up tile a down tile waits for is running or done.
template <int BN, int kStages>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_fused_kernel(const __grid_constant__ CUtensorMap tmA_gu, const __grid_constant__ CUtensorMap tmB_gu,
                              const __grid_constant__ CUtensorMap tmBsh, const __grid_constant__ CUtensorMap tmA_dn,
                              const __grid_constant__ CUtensorMap tmB_dn, const FusedArgs fa) {
  using C = Cfg<true, 2, BN, kStages>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kStages * C::kABytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + kStages * C::kBBytes);
  uint64_t* full = bars;
  uint64_t* empty = full + kStages;
  uint64_t* tfull = empty + kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_base_smem = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_smem + 1);
  const GemmArgs& gu = fa.gu;
  const GemmArgs& dn = fa.dn;

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
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == kWarpTma && lane == 0) {
    tma_prefetch_desc(&tmA_gu);
    tma_prefetch_desc(&tmB_gu);
    tma_prefetch_desc(&tmBsh);
    tma_prefetch_desc(&tmA_dn);
    tma_prefetch_desc(&tmB_dn);
  }
  if (warp == kWarpMma) {
    tmem_alloc(tmem_base_smem, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_base_smem;

  const int n_gu = *gu.ntiles;
  const int n_all = n_gu + *dn.ntiles;
  const int tfirst = static_cast<int>(blockIdx.x);
  // the tile of combined index t: gate/up tiles first, then down tiles
  auto tile_of = [&](int t, bool& is_dn) {
    is_dn = t >= n_gu;
    return load_tile<BN>(is_dn ? dn : gu, is_dn ? t - n_gu : t);
  };

  if (warp == kWarpTma) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      long issued = 0;
      bool ok = true;
      for (int t = tfirst; ok && t < n_all && !*abort_flag; t += gridDim.x) {
        bool is_dn;
        const Tile tl = tile_of(t, is_dn);
        const GemmArgs& a = is_dn ? dn : gu;
        const CUtensorMap* ma = is_dn ? &tmA_dn : &tmA_gu;
        const CUtensorMap* mb = is_dn ? &tmB_dn : (tl.group >= gu.n_routed ? &tmBsh : &tmB_gu);
        const int a_row = tl.group * a.a_rows_per_group + tl.m_tile * C::kARows;
        if (is_dn) {
          // the group's h rows: every gate/up tile of the group has stored them
          const int g = tl.group;
          const int target = fa.m_tiles_gu * ((fa.cnt[g] + BN - 1) / BN) * kEpiWarps;
          if (!wait_count(fa.done + g, target, gu, abort_flag)) break;
          fence_proxy_async_global();
        }
        const int nb = (tl.nrows + kBBoxRows - 1) / kBBoxRows;
        const uint32_t bytes = C::kABytes + nb * kBBoxBytes;
        for (int kb = 0; kb < tl.nkb; ++kb) {
          if (!wait_or_abort(&empty[stage], phase ^ 1, gu, abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[stage], bytes);
          const int kx = kb * kBK;
          tma_load_2d(sA + stage * C::kABytes, ma, &full[stage], kx, a_row, kCacheEvictFirst);
          for (int j = 0; j < nb; ++j)
            tma_load_2d(sB + stage * C::kBBytes + j * kBBoxBytes, mb, &full[stage], kx, tl.b_row0 + j * kBBoxRows,
                        kCacheEvictLast);
          ++issued;
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (*abort_flag) drain_ring(full, kStages, issued, gu.timeout_ns);
    }
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = tfirst; ok && t < n_all && !*abort_flag; t += gridDim.x) {
        bool is_dn;
        const Tile tl = tile_of(t, is_dn);
        const uint32_t n_mma = max(16, (tl.nrows + 15) & ~15);
        const uint32_t idesc = idesc_bf16_f32(128, n_mma);
        if (!wait_or_abort(&tempty[acc], acc_phase ^ 1, gu, abort_flag)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + acc * C::kAccCols;
        for (int kb = 0; kb < tl.nkb; ++kb) {
          if (!wait_or_abort(&full[stage], phase, gu, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * C::kABytes);
          const uint32_t b_addr = smem_u32(sB + stage * C::kBBytes);
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k) {
            const uint64_t bdesc = sdesc_sw128(b_addr + k * 32);
            const uint32_t accum = (kb | k) != 0;
            umma_f16(d, sdesc_sw128(a_addr + k * 32), bdesc, idesc, accum);
            umma_f16(d + BN, sdesc_sw128(a_addr + 128 * 128 + k * 32), bdesc, idesc, accum);
          }
          umma_commit(&empty[stage]);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
        if (++acc == C::kAccBufs) {
          acc = 0;
          acc_phase ^= 1;
        }
      }
      umma_commit(drain);
      const uint64_t t0 = globaltimer_ns();
      while (!mbar_try_wait(drain, 0) && globaltimer_ns() - t0 < gu.timeout_ns) {
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..)
    const int q = warp & 3;
    const int cfirst = ((warp - 2) / 4) * 16;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = tfirst; t < n_all; t += gridDim.x) {
      bool is_dn;
      const Tile tl = tile_of(t, is_dn);
      const GemmArgs& a = is_dn ? dn : gu;
      const int n_mma = max(16, (tl.nrows + 15) & ~15);
      bool ok = true;
      if (lane == 0) ok = wait_or_abort(&tfull[acc], acc_phase, gu, abort_flag);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * C::kAccCols;
      const bool rows_ok = tl.out_row0 >= 0 && tl.out_row0 + tl.nrows <= a.out_rows;
      if (!rows_ok && lane == 0 && q == 0) report_status(a.status, kStatusDevice);
      for (int c0 = cfirst; c0 < n_mma; c0 += 16 * kEpiGroups) {
        uint32_t g0[16], g1[16];
        tmem_ld16(tb + c0, g0);
        tmem_ld16(tb + BN + c0, g1);
        tmem_ld_wait();
        if (!is_dn) {
          // h = silu(min(G, L)) * clamp(U, -L, L), BF16
          const int m = tl.m_tile * 128 + q * 32 + lane;
          const bool m_ok = m < a.m_limit && rows_ok;
          __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.out);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int n = c0 + j;
            if (n < tl.nrows && m_ok) {
              const float hv = clamped_swiglu_f32(__uint_as_float(g0[j]), __uint_as_float(g1[j]), a.limit);
              out[static_cast<size_t>(tl.out_row0 + n) * a.out_ld + m] = __float2bfloat16_rn(hv);
            }
          }
        } else {
          // fp32 O rows: columns m (first 128 W2 rows of the tile) and m + 128
          const int m = tl.m_tile * 256 + q * 32 + lane;
          float* out = static_cast<float*>(a.out);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int n = c0 + j;
            if (n < tl.nrows && rows_ok) {
              const size_t o = static_cast<size_t>(tl.out_row0 + n) * a.out_ld;
              if (m < a.m_limit) out[o + m] = __uint_as_float(g0[j]);
              if (m + 128 < a.m_limit) out[o + m + 128] = __uint_as_float(g1[j]);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&tempty[acc]);
        if (!is_dn) {
          // this warp's h stores of the tile, visible GPU-wide (and to the TMA) before the count
          __threadfence();
          fence_proxy_async_global();
          atomicAdd(fa.done + tl.group, 1);
        }
      }
      if (++acc == C::kAccBufs) {
        acc = 0;
        acc_phase ^= 1;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

template <bool kGateUp, int kAMmas, int BN, int kStages>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmBsh, const GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  gemm_body<kGateUp, kAMmas, BN, kStages>(&tmA, &tmB, &tmBsh, args, smem_raw, tile_first(args),
                                          tile_count<BN>(args));
}

// The ring of the thin tiles: kThinRows-token stages, as many as fit.
template <int kAMmas>
constexpr int thin_stages() {
  return (227 * 1024 - 1024 - 512) / (kAMmas * 128 * 128 + kThinRows * 128);
}

// Two token-tile widths in one launch: the width the permutation kernel chose
// (*args.bn_select, written before this grid starts) selects the body. With
// args.thin_begin (kThinSplit) the list's thin tail is a second list: the last
// CTAs, in proportion to its estimated work (a thin tile counted as half a wide
// one), start on it with the thin ring, the others on the wide tiles, both lists
// taken through counters, and every CTA moves to the other list when its own is
// done.
template <bool kGateUp, int kAMmas, int BN1, int S1, int BN2, int S2>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_dual_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                             const __grid_constant__ CUtensorMap tmBsh, const GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  const int n = *args.ntiles;
  const bool wide2 = *args.bn_select == BN2;
  int mid = n;
  if (kThinSplit && args.thin_begin != nullptr && args.sched != nullptr) mid = min(max(*args.thin_begin, 0), n);
  if (mid == n) {
    if (wide2)
      gemm_body<kGateUp, kAMmas, BN2, S2>(&tmA, &tmB, &tmBsh, args, smem_raw, 0, n);
    else
      gemm_body<kGateUp, kAMmas, BN1, S1>(&tmA, &tmB, &tmBsh, args, smem_raw, 0, n);
    return;
  }
  if constexpr (kThinSplit) {
    const int G = static_cast<int>(gridDim.x);
    const float w_thin = 0.5f * static_cast<float>(n - mid), w_wide = static_cast<float>(mid);
    const int n_thin = mid == 0 ? G : min(max(static_cast<int>(G * w_thin / (w_thin + w_wide) + 0.5f), 1), G);
    auto wide = [&](bool again) {
      return wide2 ? gemm_body<kGateUp, kAMmas, BN2, S2>(&tmA, &tmB, &tmBsh, args, smem_raw, 0, mid, args.sched, again)
                   : gemm_body<kGateUp, kAMmas, BN1, S1>(&tmA, &tmB, &tmBsh, args, smem_raw, 0, mid, args.sched, again);
    };
    auto thin = [&](bool again) {
      return gemm_body<kGateUp, kAMmas, kThinRows, thin_stages<kAMmas>()>(&tmA, &tmB, &tmBsh, args, smem_raw, mid, n,
                                                                         args.sched + 1, again);
    };
    if (static_cast<int>(blockIdx.x) >= G - n_thin) {
      if (thin(true)) wide(false);
    } else {
      if (wide(true)) thin(false);
    }
  }
}

template <bool kGateUp, int kAMmas, int BN, int kStages>
cudaError_t set_attr() {
  return cudaFuncSetAttribute(grouped_gemm_kernel<kGateUp, kAMmas, BN, kStages>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              Cfg<kGateUp, kAMmas, BN, kStages>::kSmemBytes);
}

template <bool kGateUp, int kAMmas, int BN1, int S1, int BN2, int S2>
constexpr int dual_smem() {
  constexpr int a = Cfg<kGateUp, kAMmas, BN1, S1>::kSmemBytes, b = Cfg<kGateUp, kAMmas, BN2, S2>::kSmemBytes;
  constexpr int c = kThinSplit ? Cfg<kGateUp, kAMmas, kThinRows, thin_stages<kAMmas>()>::kSmemBytes : 0;
  return a > b ? (a > c ? a : c) : (b > c ? b : c);
}

template <bool kGateUp, int kAMmas, int BN1, int S1, int BN2, int S2>
cudaError_t set_attr_dual() {
  return cudaFuncSetAttribute(grouped_gemm_dual_kernel<kGateUp, kAMmas, BN1, S1, BN2, S2>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              dual_smem<kGateUp, kAMmas, BN1, S1, BN2, S2>());
}

template <bool kGateUp, int kAMmas, int BN, int kStages>
cudaError_t launch(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmBsh, const GemmArgs& a,
                   int grid, cudaStream_t s) {
  grouped_gemm_kernel<kGateUp, kAMmas, BN, kStages>
      <<<grid, kThreads, Cfg<kGateUp, kAMmas, BN, kStages>::kSmemBytes, s>>>(tmA, tmB, tmBsh, a);
  return cudaGetLastError();
}

template <bool kGateUp, int kAMmas, int BN1, int S1, int BN2, int S2>
cudaError_t launch_dual(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmBsh,
                        const GemmArgs& a, int grid, cudaStream_t s) {
  if (a.bn_select == nullptr) return cudaErrorInvalidValue;
  grouped_gemm_dual_kernel<kGateUp, kAMmas, BN1, S1, BN2, S2>
      <<<grid, kThreads, dual_smem<kGateUp, kAMmas, BN1, S1, BN2, S2>(), s>>>(tmA, tmB, tmBsh, a);
  return cudaGetLastError();
}

// Ring depths: as many stages of (A box + B boxes) as fit in 227 KB, unless set.
//   gate/up  BN 32: 6 x (32 + 4) KB   BN 128: 4 x (32 + 16) KB
//   down     BN 32: 10 x (16 + 4) KB, wide (256 W2 rows) 6 x (32 + 4) KB
//   large    BN 256: 3 (gate/up, wide down) or 4 (down); BN 192: 4 (gate/up, wide down)
constexpr int ring_fit(int a_bytes, int b_bytes) {
  return (227 * 1024 - 1024 - 512) / (a_bytes + b_bytes);
}
#ifndef MOE_STAGES_GU_SMALL
#define MOE_STAGES_GU_SMALL 6
#endif
#ifndef MOE_STAGES_GU_MID
#define MOE_STAGES_GU_MID 4
#endif
#ifndef MOE_STAGES_GU_LARGE
#define MOE_STAGES_GU_LARGE ring_fit(256 * 128, kBnLarge * 128)
#endif
#ifndef MOE_STAGES_DN_SMALL
#define MOE_STAGES_DN_SMALL 10
#endif
#ifndef MOE_STAGES_DN_LARGE
#define MOE_STAGES_DN_LARGE ring_fit(128 * 128, kBnLarge * 128)
#endif
#ifndef MOE_STAGES_DN_WIDE
#define MOE_STAGES_DN_WIDE ring_fit(256 * 128, kBnLarge * 128)
#endif
#define MOE_GU_SMALL true, 2, 32, MOE_STAGES_GU_SMALL
#define MOE_GU_MID true, 2, 128, MOE_STAGES_GU_MID
#define MOE_GU_LARGE true, 2, kBnLarge, MOE_STAGES_GU_LARGE
#define MOE_DN_SMALL false, 1, 32, MOE_STAGES_DN_SMALL
#define MOE_DN_LARGE false, 1, kBnLarge, MOE_STAGES_DN_LARGE
#define MOE_DN_WIDE false, 2, kBnLarge, MOE_STAGES_DN_WIDE
#define MOE_DN_WIDE_SMALL false, 2, 32, ring_fit(256 * 128, 32 * 128)
// the device-chosen alternative width (as many stages as fit), paired with the
// large width in one dual-width kernel
constexpr int kBnAltT = kBnAlt > 0 ? kBnAlt : 64;  // an unused placeholder when disabled
#define MOE_GU_DUAL true, 2, kBnLarge, MOE_STAGES_GU_LARGE, kBnAltT, ring_fit(256 * 128, kBnAltT * 128)
#define MOE_DN_WIDE_DUAL false, 2, kBnLarge, MOE_STAGES_DN_WIDE, kBnAltT, ring_fit(256 * 128, kBnAltT * 128)

}  // namespace

// the fused few-token launch: 32-token tiles, the gate/up ring depth (both halves
// have 256-row A boxes and 32-row B boxes)
#define MOE_FUSED_SMALL 32, MOE_STAGES_GU_SMALL

cudaError_t gemm_set_attributes() {
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(grouped_gemm_fused_kernel<MOE_FUSED_SMALL>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                Cfg<true, 2, MOE_FUSED_SMALL>::kSmemBytes)) != cudaSuccess)
    return e;
  if ((e = set_attr<MOE_GU_SMALL>()) != cudaSuccess) return e;
  if ((e = set_attr<MOE_GU_MID>()) != cudaSuccess) return e;
  if ((e = set_attr<MOE_GU_LARGE>()) != cudaSuccess) return e;
  if ((e = set_attr<MOE_DN_SMALL>()) != cudaSuccess) return e;
  if ((e = set_attr<MOE_DN_LARGE>()) != cudaSuccess) return e;
  if ((e = set_attr<MOE_DN_WIDE>()) != cudaSuccess) return e;
  if ((e = set_attr<MOE_DN_WIDE_SMALL>()) != cudaSuccess) return e;
  if constexpr (kBnAlt > 0) {
    if ((e = set_attr_dual<MOE_GU_DUAL>()) != cudaSuccess) return e;
    if ((e = set_attr_dual<MOE_DN_WIDE_DUAL>()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_gemm_gateup(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmBsh,
                               const GemmArgs& a, int bn, int grid, cudaStream_t s) {
  if (bn == 32) return launch<MOE_GU_SMALL>(tmA, tmB, tmBsh, a, grid, s);
  if (bn == 128) return launch<MOE_GU_MID>(tmA, tmB, tmBsh, a, grid, s);
  if (bn == kBnLarge) return launch<MOE_GU_LARGE>(tmA, tmB, tmBsh, a, grid, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_gemm_down(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& a, int bn, int grid,
                             cudaStream_t s, bool wide) {
  if (wide) {
    if (bn == kBnLarge) return launch<MOE_DN_WIDE>(tmA, tmB, tmB, a, grid, s);
    if (bn == 32) return launch<MOE_DN_WIDE_SMALL>(tmA, tmB, tmB, a, grid, s);
    return cudaErrorInvalidValue;
  }
  if (bn == 32) return launch<MOE_DN_SMALL>(tmA, tmB, tmB, a, grid, s);
  if (bn == kBnLarge) return launch<MOE_DN_LARGE>(tmA, tmB, tmB, a, grid, s);
  return cudaErrorInvalidValue;
}

}  // namespace moe

namespace moe {

cudaError_t launch_gemm_gateup_dual(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmBsh,
                                    const GemmArgs& a, int grid, cudaStream_t s) {
  if constexpr (kBnAlt > 0) return launch_dual<MOE_GU_DUAL>(tmA, tmB, tmBsh, a, grid, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_gemm_down_wide_dual(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& a, int grid,
                                       cudaStream_t s) {
  if constexpr (kBnAlt > 0) return launch_dual<MOE_DN_WIDE_DUAL>(tmA, tmB, tmB, a, grid, s);
  return cudaErrorInvalidValue;
}

}  // namespace moe

namespace moe {

cudaError_t launch_gemm_fused_small(const CUtensorMap& tmA_gu, const CUtensorMap& tmB_gu, const CUtensorMap& tmBsh,
                                   const CUtensorMap& tmA_dn, const CUtensorMap& tmB_dn, const FusedArgs& f,
                                   int grid, cudaStream_t s) {
  // cooperative: every CTA resident at once (a down tile waits for other CTAs' gate/up tiles)
  void* args[] = {const_cast<CUtensorMap*>(&tmA_gu), const_cast<CUtensorMap*>(&tmB_gu),
                  const_cast<CUtensorMap*>(&tmBsh),  const_cast<CUtensorMap*>(&tmA_dn),
                  const_cast<CUtensorMap*>(&tmB_dn), const_cast<FusedArgs*>(&f)};
  return cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(grouped_gemm_fused_kernel<MOE_FUSED_SMALL>),
                                     dim3(grid), dim3(kThreads), args, Cfg<true, 2, MOE_FUSED_SMALL>::kSmemBytes, s);
}

}  // namespace moe
