/*
 * moe.h - C ABI of the B200 (sm_100a) DeepSeek-V4.1-Flash routed-expert FFN layer.
 *
 * The layer (DeepSeek V4.1 inference/config.json: "n_routed_experts" 384,
 * "n_shared_experts" 1, "n_activated_experts" 6, "dim" 5120, "moe_inter_dim"
 * 2304, "score_func" "sqrtsoftplus", "route_scale" 1.5, "swiglu_limit" 10.0,
 * "expert_dtype" "fp4"; MAX DeepseekV41Config fields of the same meaning):
 *
 *   z_e  = x . Wg_e (+ b_e)                     router logits, e < E
 *   s_e  = sqrt(softplus(z_e))                  "sqrtsoftplus" score
 *   sel  = the top_k experts by s_e (ties: lower index first), descending
 *   w_j  = route_scale * s_sel(j) / sum_j s_sel(j)
 *   f(x) = W2 (silu(min(W1 x, L)) * clamp(W3 x, -L, L)),   L = swiglu_limit
 *   y    = sum_{shared} f_sh(x) + sum_j w_j f_sel(j)(x)
 *
 * The pages name the score function and the clamp but print no formula; the
 * lines above are the plainest reading and the one the library computes.
 *
 * Conventions for every entry point
 *   - Device pointers are CUDA device (or managed) addresses on the device that
 *     was current when the handle was created; host pointers are noted as such.
 *   - Every matrix is row-major [out, in]: the input (reduction) dimension is
 *     contiguous. BF16 is IEEE bfloat16 bit patterns in uint16 storage.
 *   - A stream argument is a cudaStream_t (NULL = legacy default stream). Work is
 *     enqueued on it and the call returns without synchronising unless the entry
 *     point says otherwise.
 *   - Argument errors are detected before anything is enqueued and returned as a
 *     status; no entry point aborts the process or prints.
 *   - Device-side bounded waits that run out record MOE_ERR_TIMEOUT in the
 *     handle's status word, read by moe_get_status().
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MOE_ABI_VERSION 4

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

struct CUstream_st;
typedef struct CUstream_st* moe_stream_t; /* == cudaStream_t */

typedef struct moe_handle moe_handle;

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1, /* null pointer, bad size, T > max_tokens, misaligned pointer */
  MOE_ERR_UNSUPPORTED = 2, /* valid but outside what the kernels implement (see moe_config) */
  MOE_ERR_OOM = 3,         /* device allocation failed inside moe_create */
  MOE_ERR_CUDA = 4,        /* a CUDA runtime call or kernel launch failed */
  MOE_ERR_TIMEOUT = 5,     /* a device-side bounded wait ran out (reported by moe_get_status) */
  MOE_ERR_DEVICE = 6       /* a device-side consistency check failed (reported by moe_get_status) */
} moe_status;

typedef enum {
  MOE_DT_BF16 = 0, /* routed experts in BF16 */
  MOE_DT_MXFP4 = 1, /* routed experts in MXFP4: E2M1 values + one E8M0 scale per 32 along K */
  MOE_DT_MXFP8 = 2  /* routed experts in MXFP8: E4M3 values + one E8M0 scale per 32 along K (the
                       checkpoint's "dtype": "fp8" and MAX's float8_e4m3fn encoding; the pages give no
                       FP8 scale granularity, so the block is the family's E8M0-per-32) */
} moe_expert_dtype;

/*
 * Layer shape and constants (MAX DeepseekV41Config: hidden_size,
 * moe_intermediate_size, n_routed_experts, n_shared_experts,
 * num_experts_per_tok, routed_scaling_factor, swiglu_limit).
 *
 * Supported: hidden % 128 == 0, inter % 128 == 0, both <= 16384,
 * 1 <= top_k <= min(n_routed, 32), n_routed <= 512 (the top-k kernels hold up
 * to 16 scores per lane and 32 selections per token in registers),
 * 0 <= n_shared <= 4, 1 <= max_tokens <= 65536, route_scale > 0 and finite,
 * swiglu_limit >= 0 (INFINITY disables both clamps). Anything else returns
 * MOE_ERR_UNSUPPORTED (shape) or MOE_ERR_INVALID_ARG (NaN, negative, zero).
 */
typedef struct {
  int32_t hidden;       /* H */
  int32_t inter;        /* I, expert width (routed and shared) */
  int32_t n_routed;     /* E */
  int32_t n_shared;     /* shared experts, weight 1 each */
  int32_t top_k;        /* k */
  int32_t max_tokens;   /* largest T a forward may pass; sizes the workspace */
  float route_scale;    /* rho */
  float swiglu_limit;   /* L */
  int32_t expert_dtype; /* moe_expert_dtype of the routed experts */
} moe_config;

/*
 * Weights, all device pointers, read during moe_create only (the library keeps
 * its own repacked copy; the caller may free its buffers once the create
 * stream has completed).
 *   router_w     BF16 [E, H]
 *   router_bias  fp32 [E] added to the logits (selection and weights), or NULL
 *   BF16 experts:  w1, w3 BF16 [E, I, H]; w2 BF16 [E, H, I]; s1 = s3 = s2 = NULL
 *   MXFP4 experts: w1, w3 uint8 [E, I, H/2]; w2 uint8 [E, H, I/2]: E2M1 pairs,
 *                  element 2j in the low nibble of byte j (float4_e2m1fnx2);
 *                  s1, s3 uint8 [E, I, H/32]; s2 uint8 [E, H, I/32]: E8M0
 *                  scales (2^(code-127)), code 0xFF (NaN) is rejected.
 *   MXFP8 experts: w1, w3 uint8 [E, I, H]; w2 uint8 [E, H, I]: E4M3 codes
 *                  (float8_e4m3fn); s1, s3, s2 E8M0 scales as for MXFP4.
 *   With MXFP4 or MXFP8 experts the routed experts see the token and their
 *   SwiGLU output quantised to MXFP8 (E4M3, E8M0 per 32, OCP MX v1.0 rule);
 *   the router and the shared experts see BF16.
 *   sh_w1, sh_w3 BF16 [n_shared, I, H]; sh_w2 BF16 [n_shared, H, I] (always BF16)
 * Every pointer must be 16-byte aligned.
 */
typedef struct {
  const void* router_w;
  const float* router_bias;
  const void* w1;
  const void* w3;
  const void* w2;
  const uint8_t* s1;
  const uint8_t* s3;
  const uint8_t* s2;
  const void* sh_w1;
  const void* sh_w3;
  const void* sh_w2;
} moe_weights;

/*
 * Create a layer on the current device: validate, allocate the repacked
 * weights and the workspace for cfg->max_tokens tokens, and enqueue the weight
 * repack on `stream` (the analogue of the MAX pipeline's one-time routed-expert
 * upload, DeepseekV41Model.load_model). On success *out owns all device memory
 * it allocated. On failure *out is NULL and nothing is leaked. (For tests of
 * that path: with the environment variable MOE_TEST_FAIL_ALLOC_AFTER=n set, the
 * create makes its (n+1)-th device allocation fail.) Every weight
 * pointer must be device (or managed) memory of the current device, else
 * MOE_ERR_INVALID_ARG before anything is enqueued.
 */
MOE_API moe_status moe_create(const moe_config* cfg, const moe_weights* w, moe_stream_t stream,
                      moe_handle** out);

/*
 * One layer invocation on T token rows.
 *   x        BF16 [T, H] device, 16-byte aligned
 *   y        BF16 [T, H] device, 16-byte aligned (may not alias x)
 *   topk_idx int32 [T, k] device or NULL: selected experts, descending score
 *   topk_w   fp32  [T, k] device or NULL: their weights (sum = route_scale)
 * 0 <= T <= max_tokens; T == 0 enqueues nothing. Allocates nothing and does not
 * synchronise. A token whose router scores are not finite (NaN or infinite
 * input) gets placeholder experts with NaN weights and a NaN output row, and
 * moe_get_status then reports MOE_ERR_DEVICE; other tokens are unaffected. Calls on one handle must be ordered (one stream at a time): the
 * workspace is shared between calls. MOE_ERR_INVALID_ARG, with nothing enqueued,
 * when the current device is not the handle's or x / y are not device (or
 * managed) memory of it (a host pointer would fault the kernels).
 */
MOE_API moe_status moe_forward(moe_handle* h, const void* x, int32_t T, void* y, int32_t* topk_idx,
                       float* topk_w, moe_stream_t stream);

/*
 * Expert parallelism (MAX DeepseekV41Config ep_config, "only under data
 * parallelism"; the DEP recipes on the DeepSeek-V4-Pro page). The routed
 * experts are split into windows, one per rank; every rank keeps the whole
 * router. A rank routes all the ranks' tokens (gathered), runs only the slots
 * whose expert lies in its window, and produces a partial output; the partial
 * outputs of a partition of [0, n_routed) sum to the layer's output. The
 * collectives (all-gather of x, reduce-scatter of the partial outputs) are the
 * caller's (the Python package's ExpertParallelLayer uses torch.distributed).
 *
 * moe_create_ep: as moe_create, holding routed experts [expert_begin,
 * expert_begin + expert_count) of cfg->n_routed. router_w [n_routed, H] and
 * router_bias [n_routed] are whole; w1 / w3 / w2 (and s1 / s3 / s2) hold the
 * window's expert_count experts only. The shared experts are cfg->n_shared
 * of them on this rank (give them to exactly one rank, 0 to the others).
 *
 * moe_forward_partial: y_partial fp32 [T, H] device = this instance's share:
 * sum over the selected slots of its window of w_j f_j(x), plus its shared
 * experts, summed in fp32 in slot order and not rounded. Works on any handle
 * (a whole layer gives the full output in fp32). moe_forward and
 * moe_forward_hashed reject a handle that holds a window of the experts
 * (MOE_ERR_INVALID_ARG).
 */
MOE_API moe_status moe_create_ep(const moe_config* cfg, const moe_weights* w, int32_t expert_begin,
                                 int32_t expert_count, moe_stream_t stream, moe_handle** out);
MOE_API moe_status moe_forward_partial(moe_handle* h, const void* x, int32_t T, float* y_partial,
                                       int32_t* topk_idx, float* topk_w, moe_stream_t stream);

/*
 * Hash-routed layers (MAX DeepseekV41Config num_hash_layers; DeepSeek-V4-Pro has
 * 3). The pages name them but give no hash function; this library reads them
 * as: token t takes the top_k experts of row token_ids[t] of a fixed vocabulary
 * table, in the row's order, in place of the router's top-k; the weights are
 * the sqrtsoftplus scores of those experts (router logits + bias as for learned
 * routing) normalised over the top_k and scaled by route_scale. Everything after
 * the routing is the same layer.
 *
 * moe_set_hash_table: table int32 [vocab, top_k] device, every entry in
 * [0, n_routed) and no expert twice in a row, else MOE_ERR_INVALID_ARG (the
 * check runs on `stream`, and this call synchronises it). The library keeps
 * its own copy (the only device allocation after moe_create; MOE_ERR_OOM if it
 * fails); a later call replaces the table.
 *
 * moe_forward_hashed: as moe_forward, with token_ids int32 [T] device (the
 * tokens' vocabulary ids). MOE_ERR_INVALID_ARG when no table was set. An id
 * outside [0, vocab) gives that token the placeholder experts 0..top_k-1 with
 * NaN weights and a NaN output row, and moe_get_status reports MOE_ERR_DEVICE.
 */
MOE_API moe_status moe_set_hash_table(moe_handle* h, const int32_t* table, int32_t vocab, moe_stream_t stream);
MOE_API moe_status moe_forward_hashed(moe_handle* h, const void* x, const int32_t* token_ids, int32_t T, void* y,
                                      int32_t* topk_idx, float* topk_w, moe_stream_t stream);

/*
 * moe_forward on HOST buffers: copies x (BF16 [T, H], host, ideally pinned)
 * into a handle-owned device staging buffer, runs the layer, and copies y
 * (and topk_idx / topk_w when not NULL, host [T, k]) back, all enqueued on
 * `stream`. The host buffers must stay valid until the stream reaches the end
 * of the copies; synchronise the stream before reading them.
 */
MOE_API moe_status moe_forward_host(moe_handle* h, const void* x_host, int32_t T, void* y_host,
                            int32_t* topk_idx_host, float* topk_w_host, moe_stream_t stream);

/*
 * Pipelined host path for a stream of batches: like moe_forward_host (x_host
 * BF16 [T, hidden], y_host BF16 [T, hidden], both host memory, pinned for the
 * copies to overlap), but the copies run on two internal streams. The layer is
 * enqueued on `stream` after its x has arrived, and y leaves on the copy-out
 * stream. So the copy of the next call's x and the copy-out of the previous call's
 * y overlap this call's layer. Two device staging slots alternate between calls
 * (the second is allocated on the first call: MOE_ERR_OOM if that fails).
 * Ordering: x_host is read without waiting for earlier work on `stream`, and y_host
 * is written without ordering against later work on `stream`. Call
 * moe_forward_host_wait(h, stream) and then synchronise `stream` before reading
 * any y_host, or reusing an x_host or y_host of a call that may still be in flight
 * (at most the last two calls). Routing indices are not copied; hash layers and
 * expert-window handles are not supported (MOE_ERR_INVALID_ARG, from moe_forward).
 */
MOE_API moe_status moe_forward_host_async(moe_handle* h, const void* x_host, int32_t T, void* y_host,
                                  moe_stream_t stream);

/* Make `stream` wait for every copy-out of moe_forward_host_async so far. */
MOE_API moe_status moe_forward_host_wait(moe_handle* h, moe_stream_t stream);

/* Synchronise the device, then report and clear the device-side status word
 * (MOE_OK, MOE_ERR_TIMEOUT or MOE_ERR_DEVICE); MOE_ERR_CUDA if the sync failed. */
MOE_API moe_status moe_get_status(moe_handle* h);

/* Static string for a status code. */
MOE_API const char* moe_status_string(moe_status s);

/* Free everything the handle owns (synchronises the device first). NULL is a no-op. */
MOE_API void moe_destroy(moe_handle* h);

/* MOE_ABI_VERSION of the loaded library. */
MOE_API int32_t moe_abi_version(void);

/* ------------------------------------------------------------------------
 * Utilities (not part of the layer's arithmetic path)
 * ---------------------------------------------------------------------- */

/*
 * Quantise BF16 [rows, cols] (device) to MXFP4 with the OCP MX v1.0 rule: per
 * block of 32 along cols, scale = 2^(floor(log2(amax)) - 2) clamped to the E8M0
 * range (all-zero block: code 0), elements rounded to nearest-even E2M1 and
 * saturated at +-6. Writes packed [rows, cols/2] (low nibble = even element)
 * and scales [rows, cols/32]. cols % 32 == 0. Enqueued on `stream`.
 */
MOE_API moe_status moe_quantize_mxfp4(const void* src_bf16, int64_t rows, int32_t cols, uint8_t* dst_packed,
                              uint8_t* dst_scales, moe_stream_t stream);

/*
 * Quantise BF16 [rows, cols] (device) to MXFP8 with the same OCP MX v1.0 rule
 * and E4M3 elements: per block of 32 along cols, scale = 2^(floor(log2(amax)) - 8)
 * clamped to the E8M0 range (all-zero block: code 0), elements rounded to
 * nearest-even E4M3 and saturated at +-448. Writes codes [rows, cols] and scales
 * [rows, cols/32]. cols % 32 == 0; src and dst_codes 16-byte aligned. Enqueued
 * on `stream`.
 */
MOE_API moe_status moe_quantize_mxfp8(const void* src_bf16, int64_t rows, int32_t cols, uint8_t* dst_codes,
                              uint8_t* dst_scales, moe_stream_t stream);

/* Internal buffers of the LAST forward that moe_inspect can copy out. */
typedef enum {
  MOE_BUF_LOGITS = 0,   /* fp32 [T, E] router logits before refinement (approximate) */
  MOE_BUF_TOPK_IDX = 1, /* int32 [T, k] */
  MOE_BUF_TOPK_W = 2,   /* fp32 [T, k] */
  MOE_BUF_COUNTS = 3,   /* int32 [E + n_shared] rows per group (routed experts, then shared) */
  MOE_BUF_OFFSETS = 4,  /* int32 [E + n_shared + 1] first row of each group */
  MOE_BUF_PERM = 5,     /* int32 [T*k] flat slot t*k+j of each routed row (expert-major) */
  MOE_BUF_INV = 6,      /* int32 [T*k] row of each flat slot */
  MOE_BUF_H = 7,        /* BF16 [T*k + n_shared*T, I] SwiGLU output rows (group order) */
  MOE_BUF_XQ = 8,       /* MXFP4 / MXFP8 layers: uint8 E4M3 [T*k, H], MXFP8 codes of the routed rows (perm order) */
  MOE_BUF_XQ_SCALES = 9, /* MXFP4 / MXFP8 layers: their E8M0 scales, packed in 512-byte atoms per token tile */
  MOE_BUF_HQ = 10,       /* MXFP4 / MXFP8 layers: uint8 E4M3 [T*k, I], MXFP8 codes of the routed SwiGLU rows
                            (group order, as MOE_BUF_H) */
  MOE_BUF_HQ_SCALES = 11, /* MXFP4 / MXFP8 layers: their E8M0 scales in 512-byte atoms, one per (down-GEMM
                            token tile nt, 128-wide slice c of I): row n of the tile, block b of the
                            slice at byte (nt * I/128 + c) * 512 + (n % 32) * 16 + (n / 32) * 4 + b.
                            Token tiles: each routed group's rows cut into tiles of 32 rows when
                            T <= 32, 96 rows when T * top_k >= 24 * n_routed, else 64 rows,
                            numbered group by group in expert order */
  MOE_BUF_NTILES = 12,   /* int32 [7]: tiles in the gate/up and down lists, where their shared-expert
                            tiles end, the routed rows this instance holds, and where each list's
                            thin tail begins (partial tiles of at most 32 rows, last in a list
                            ordered longest first; the list's length when it is not ordered so) */
  MOE_BUF_TILES_GU = 13, /* int32 [n, 4] gate/up tile list: {group | m_tile << 16, B row or token-tile id,
                            first output row, rows} in the order the persistent CTAs take them */
  MOE_BUF_TILES_DN = 14  /* int32 [n, 4] the same for the down GEMM */
} moe_buffer;

/*
 * Copy `bytes` from the start of internal buffer `what` to dst (host or device;
 * cudaMemcpyAsync with cudaMemcpyDefault on `stream`). bytes must not exceed the
 * buffer's size for max_tokens. For tests and debugging.
 */
MOE_API moe_status moe_inspect(moe_handle* h, int32_t what, void* dst, size_t bytes, moe_stream_t stream);

/*
 * Fill every per-forward scratch buffer of the handle with `byte_value` (0-255;
 * 0xFF makes every float a NaN and every index -1) on `stream`, leaving the
 * status word alone. A forward must give the same bits after this as before it:
 * nothing it reads is left over from an earlier call. For tests and debugging.
 */
MOE_API moe_status moe_fill_workspace(moe_handle* h, int32_t byte_value, moe_stream_t stream);

/*
 * Read-only streaming bandwidth of the current device, in GB/s (the roofline
 * denominator of the weight-streaming kernels, which read without writing):
 * one CTA per SM keeps six 32 KiB bulk copies (global -> shared memory) in
 * flight over the whole of buf, reps times after one warm-up pass, timed with
 * CUDA events on `stream`; synchronises. buf: device memory of at least 1 MiB,
 * 16-byte aligned (far larger than L2 for a DRAM figure); bytes beyond a whole
 * number of 32 KiB chunks are not read. Allocates a 4-byte status word.
 */
MOE_API moe_status moe_read_bandwidth(const void* buf, size_t bytes, int32_t reps, moe_stream_t stream, double* gbs);

/* Limit, in nanoseconds, of every device-side wait of this handle's kernels
 * (default 2e9). A smaller value makes a stuck wait return sooner. */
MOE_API moe_status moe_set_wait_timeout(moe_handle* h, uint64_t timeout_ns);

/*
 * Launch one kernel whose only job is an mbarrier wait that nothing completes,
 * bounded by timeout_ns; it records MOE_ERR_TIMEOUT in the handle's status word
 * and returns. Proves the bounded-wait path without hanging the device.
 */
MOE_API moe_status moe_selftest_wait_timeout(moe_handle* h, uint64_t timeout_ns, moe_stream_t stream);

/* Sizes of what the handle owns. */
typedef struct {
  uint64_t weight_bytes;     /* repacked router + expert weights */
  uint64_t workspace_bytes;  /* per-forward scratch for max_tokens */
  int32_t num_sms;           /* SMs the persistent kernels are sized for */
  int32_t last_tokens;       /* T of the last forward */
} moe_info;

MOE_API moe_status moe_get_info(moe_handle* h, moe_info* out);

/*
 * Per-kernel device timing. moe_profile_begin(h, max_calls) makes the next
 * max_calls forwards record a CUDA event pair around every kernel they launch
 * (on the forward's stream). moe_profile_end(h, ms, launches, n) synchronises,
 * adds up the elapsed time per kernel kind over the recorded forwards into
 * ms[0..n) and the launch counts into launches[0..n), and stops recording.
 * Kinds are indexed as moe_kernel_name() names them.
 */
MOE_API moe_status moe_profile_begin(moe_handle* h, int32_t max_calls);
MOE_API moe_status moe_profile_end(moe_handle* h, double* ms, int64_t* launches, int32_t n);
MOE_API int32_t moe_num_kernel_kinds(void);
MOE_API const char* moe_kernel_name(int32_t kind);

/* ------------------------------------------------------------------------
 * Routing without device allocation
 * ---------------------------------------------------------------------- */

/*
 * Routing alone (router logits, sqrtsoftplus scores, top-k and the
 * route_scale-normalised weights) for callers that cannot allocate device
 * memory: code whose device memory all belongs to a host framework's pool (a
 * raw cudaMalloc there can fail or fragment that pool), loops that forbid any
 * allocation once they have started, and callers that cannot accept the
 * device-wide synchronisation cudaMalloc or cudaFree may cause. The pages have
 * no counterpart of this entry point; it is an addition of this library.
 *
 *   x           BF16 [T, hidden], device, 16-byte aligned
 *   router_w    BF16 [n_routed, hidden], device, 16-byte aligned
 *   router_bias fp32 [n_routed] device, or NULL
 *   topk_idx    int32 [T, top_k] device (output), descending score
 *   topk_w      fp32  [T, top_k] device (output), sum = route_scale
 * hidden % 8 == 0, 1 <= top_k <= min(n_routed, 32), n_routed <= 512. The
 * selection is the same as moe_forward's topk_idx for the same inputs (both
 * re-score the near-tie candidates exactly; only an exact tie of the float64
 * scores could resolve differently) and the weights agree within float32
 * rounding. Buffers that are not device (or managed) memory of the current
 * device give MOE_ERR_INVALID_ARG with nothing enqueued.
 *
 * There is no handle and so no status word: a token whose scores are not
 * finite (NaN or infinite x, router weights or bias) gets the placeholder
 * experts 0, 1, ..., top_k - 1 in the slots that found no valid expert, with
 * NaN weights; check topk_w for NaN when the input may be non-finite.
 *
 * The only scratch, the fp32 logits [T, n_routed], lives in a fixed array of
 * MOE_NOALLOC_MAX_LOGITS floats (4 MiB) inside the library; every GPU that
 * loads the library holds it until the process exits. T * n_routed above
 * MOE_NOALLOC_MAX_LOGITS returns MOE_ERR_UNSUPPORTED and enqueues nothing.
 * Nothing is allocated, by this call or by anything it calls. The first call
 * on a device looks up the array's device address once for that device (with
 * that device current); make that first call before any stream capture. The
 * looked-up address is kept for the life of the process: after
 * cudaDeviceReset (or anything else that destroys the device's primary
 * context) it is stale, so do not call this entry point on that device again
 * in the same process. All
 * calls share the one array, and each call writes every entry it later reads,
 * so nothing needs clearing between calls; calls that overlap on the GPU (on
 * streams not ordered with each other) race on it.
 */
#define MOE_NOALLOC_MAX_LOGITS (1 << 20)

MOE_API moe_status moe_route_noalloc(const void* x, const void* router_w, const float* router_bias, int32_t T,
                                     int32_t hidden, int32_t n_routed, int32_t top_k, float route_scale,
                                     int32_t* topk_idx, float* topk_w, moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
