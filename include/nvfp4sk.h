/*
 * nvfp4sk.h -- C ABI of libnvfp4sk, the B200 (sm_100a) kernels of the
 * tree-MTP verification forward step of a 27B-class dense LLM:
 *   W4A4 NVFP4 linear layers at M = 1..16 query tokens (LM head included),
 *   tree-masked attention of the draft nodes over an FP8 paged KV cache,
 *   and the page gather that restores a cached prompt prefix.
 *
 * The operations are those of "TensorRT Edge-LLM Completes the MLPerf Edge
 * Agentic Benchmark 6.4x Faster on Jetson AGX Thor" (spbcomputers.ru,
 * mechatronicstore.cl and ai4snews copies of the NVIDIA post):
 *   - section "NVFP4 and FP8: smaller weights, faster decoding": low-batch
 *     decode is DRAM-bandwidth bound; weights AND activations are NVFP4,
 *     the LM head included; the KV cache is FP8;
 *   - section "KV-cache reuse between agent steps": a prompt prefix seen before
 *     is detected and its KV pages are copied back from the cache;
 *   - section "Tree multi-token prediction": candidates are organised into a
 *     16-node tree (8 draft steps, top-2 per depth) and verified in ONE
 *     forward pass of the target model.
 * Codec definitions: E2M1 per OCP Microscaling Formats (MX) v1.0, E4M3 per
 * OCP 8-bit Floating Point Specification (OFP8, "fn" variant, max 448).
 *
 * Conventions for every call
 *   - All tensor arguments are DEVICE pointers to caller-owned memory unless
 *     stated otherwise; the library allocates nothing per call.
 *   - Calls are asynchronous on `stream` (a cudaStream_t) and return before
 *     the GPU work ends.  Host-side argument checks return an error code and
 *     launch nothing; they run before the current device is looked up, so a
 *     bad argument reports the same code with or without a usable GPU, and a
 *     well-formed call without an sm_100 device returns NVFP4SK_ERR_DEVICE
 *     (or NVFP4SK_ERR_CUDA when no device is visible).  Device-side problems (a page id out of range, a wait
 *     that ran out) never trap: the kernel skips the access, records the
 *     problem in a device error word and returns; nvfp4sk_get_device_status()
 *     reports and clears it.
 *   - A "workspace" is caller-owned device scratch of at least the size the
 *     matching *_workspace_bytes() query returns.  The nvfp4_linear,
 *     argmax_rows_bf16 and tree_attn_fp8kv workspaces start with arrival
 *     counters that must read zero when a call starts: zero-fill such a
 *     workspace once when it is allocated and do not lend it to another kind
 *     of call (nvfp4_quantize_act leaves partial results in its own); every
 *     successful call leaves its counters zero again.  A call whose device
 *     status later reads non-zero (a wait that ran out, above all) may leave
 *     counters non-zero: after nvfp4sk_get_device_status returns an error,
 *     zero every nvfp4_linear, argmax_rows_bf16 and tree_attn_fp8kv workspace
 *     again before its next use (the ctypes binding does this for its
 *     default workspaces).
 *     Calls that share one workspace must be stream-ordered.
 *   - Scalars such as tensor scales are device pointers, so no call syncs.
 *   - Error codes are negative; nvfp4sk_last_error() gives a message for the
 *     last failing call of the calling thread.
 */
#ifndef NVFP4SK_H
#define NVFP4SK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define NVFP4SK_API __attribute__((visibility("default")))
#else
#define NVFP4SK_API
#endif

typedef struct CUstream_st *nvfp4sk_stream_t; /* same type as cudaStream_t */
typedef int nvfp4sk_status;

#define NVFP4SK_OK 0
#define NVFP4SK_ERR_INVALID_ARG (-1)       /* null pointer, bad dtype, bad tree     */
#define NVFP4SK_ERR_UNSUPPORTED_SHAPE (-2) /* shape outside what the kernels cover  */
#define NVFP4SK_ERR_MISALIGNED (-3)        /* pointer/stride not 16-byte aligned    */
#define NVFP4SK_ERR_WORKSPACE (-4)         /* workspace missing or too small        */
#define NVFP4SK_ERR_CUDA (-5)              /* a CUDA runtime/driver call failed     */
#define NVFP4SK_ERR_TIMEOUT (-6)           /* a device wait ran out (device status) */
#define NVFP4SK_ERR_OUT_OF_RANGE (-7)      /* a device bounds check failed          */
#define NVFP4SK_ERR_DEVICE (-8)            /* current device is not sm_100          */

enum { NVFP4SK_BF16 = 0, NVFP4SK_FP32 = 1 };

/* ------------------------------------------------------------------------
 * nvfp4_quantize_act -- NVFP4 quantisation of an activation (or weight)
 * tensor (section "NVFP4 and FP8": NVFP4 for weights and activations).
 *
 * x: rows x K elements of type x_dtype (NVFP4SK_BF16 or NVFP4SK_FP32), row
 *    stride ld_x elements.  K % 16 == 0, ld_x >= K, x 16-byte aligned and
 *    ld_x * element size a multiple of 16 bytes.
 * g_in: device fp32 tensor scale, or NULL for the dynamic per-tensor scale
 *    g = fp32(amax(|x|) / 2688) (g = 1 when x is all zero).  g must be > 0.
 * Per 16-element block b of a row: r = fp32(amax_b / 6), t = fp32(r / g),
 *    scale = E4M3(t) (round-to-nearest-even, saturating at 448),
 *    s = fp32(value(scale) * g), code_k = s == 0 ? +0 : E2M1(fp32(x_k / s))
 *    (round-to-nearest-even, saturating at 6, sign kept).
 * Outputs (codes + scales, and/or act_prepared):
 *   codes:  u8 [rows][K/2], two codes per byte, even k in the low nibble.
 *   scales: u8 [rows][K/16] E4M3 (canonical row-major layout).
 *   g_out:  device fp32, receives g (may equal g_in).
 *   act_prepared: NULL, or the same codes and scales in the tile image that
 *     nvfp4_linear streams (nvfp4_prepared_act_bytes(K) bytes, 16-byte
 *     aligned, zero-filled once at allocation; needs rows <= 16, K % 64 == 0).
 * ws: workspace of nvfp4_quantize_workspace_bytes(rows, K) bytes.
 * ---------------------------------------------------------------------- */
NVFP4SK_API size_t nvfp4_quantize_workspace_bytes(int64_t rows, int64_t K);
NVFP4SK_API size_t nvfp4_prepared_act_bytes(int64_t K);
NVFP4SK_API nvfp4sk_status nvfp4_quantize_act(const void *x, int x_dtype, int64_t rows, int64_t K, int64_t ld_x,
                                              const float *g_in, uint8_t *codes, uint8_t *scales, float *g_out,
                                              uint8_t *act_prepared, void *ws, size_t ws_bytes,
                                              nvfp4sk_stream_t stream);

/* Re-layout of canonical NVFP4 activation codes [rows][K/2] and scales
 * [rows][K/16] (e.g. quantised elsewhere) into act_prepared, byte-identical to
 * what nvfp4_quantize_act writes there.  rows <= 16, K % 64 == 0. */
NVFP4SK_API nvfp4sk_status nvfp4_prepare_act(const uint8_t *codes, const uint8_t *scales, int64_t rows, int64_t K,
                                             uint8_t *act_prepared, nvfp4sk_stream_t stream);

/* ------------------------------------------------------------------------
 * nvfp4_prepare_weight -- one-time rearrangement of an NVFP4 weight (codes
 * [N][K/2], canonical E4M3 scales [N][K/16]) into the tile image that
 * nvfp4_linear streams: per 128-row x 512-K unit, 32 KB of 128-byte-swizzled
 * codes followed by 4 KB of tensor-memory scale images, contiguous.  Offline
 * step for the NVFP4 weights of section "NVFP4 and FP8" (calibrated once,
 * then served).  prepared: nvfp4_prepared_weight_bytes(N, K) bytes, 16-byte
 * aligned (opaque).  K % 64 == 0; rows/columns beyond N/K are zero-padded.
 * codes must be 16-byte aligned and scales 4-byte aligned.  Also the tile
 * image of a many-token activation for nvfp4_linear_wide (tokens as rows).
 * ---------------------------------------------------------------------- */
NVFP4SK_API size_t nvfp4_prepared_weight_bytes(int64_t N, int64_t K);
NVFP4SK_API nvfp4sk_status nvfp4_prepare_weight(const uint8_t *codes, const uint8_t *scales, int64_t N, int64_t K,
                                                uint8_t *prepared, nvfp4sk_stream_t stream);

/* ------------------------------------------------------------------------
 * nvfp4_linear -- the W4A4 NVFP4 linear layer of the verify step at
 * M = 1..16 tokens, LM head included (section "NVFP4 and FP8": low-batch
 * decode is DRAM-bandwidth bound; weights, activations and the LM head are
 * NVFP4).  Y[m][n] = bf16( g_a*g_w * sum_b s_a[m,b] s_w[n,b] sum_{k in b}
 * a[m,k] w[n,k]  (+ residual[m][n]) ), fp32 accumulation on tcgen05
 * block-scaled tensor cores, split-K across all SMs.
 *
 * a_prepared, g_a: activation from nvfp4_quantize_act (act_prepared) or the
 *   fused quantisers; 1 <= M <= 16 rows.
 * w_prepared, g_w: weight from nvfp4_prepare_weight (+ its tensor scale).
 *   With programmatic dependent launch on (the default) the first weight
 *   units are requested before the preceding kernel on the stream has
 *   finished, and the kernel lets its own dependents start at once: the
 *   weights must not be written by a kernel that may still run (see
 *   tree_attn_fp8kv for the rule).
 * K % 64 == 0, 1 <= N <= 524288; prepared operands 16-byte aligned.
 * residual: NULL or bf16 [M][ldy] added before rounding (may alias y).
 * y: bf16 [M][ldy], ldy >= N.
 * ws: nvfp4_linear_workspace_bytes(M, N, K) bytes, zero-filled at allocation
 *   and again after a failing device status (the workspace rule above).
 * ---------------------------------------------------------------------- */
NVFP4SK_API size_t nvfp4_linear_workspace_bytes(int64_t M, int64_t N, int64_t K);
NVFP4SK_API nvfp4sk_status nvfp4_linear(const uint8_t *a_prepared, const float *g_a, int64_t M,
                                        const uint8_t *w_prepared, const float *g_w, int64_t N, int64_t K,
                                        const void *residual, void *y, int64_t ldy, void *ws, size_t ws_bytes,
                                        nvfp4sk_stream_t stream);

/* ------------------------------------------------------------------------
 * nvfp4_linear_swiglu -- the gate+up linear of the verify step with the
 * SwiGLU and its NVFP4 quantisation in the epilogue (the down linear's input;
 * section "NVFP4 and FP8": activations are NVFP4, here with a calibrated
 * static tensor scale).  For f < F and m < M, with gate = row f and up = row
 * F + f of the [2F, K] weight:
 *   gu[m][f]  = bf16( g_a*g_w * sum ... )      (what nvfp4_linear would store)
 *   s[m][f]   = bf16( silu(gu_gate) * gu_up )   (silu(x) = x / (1 + exp(-x)))
 *   act_out   = NVFP4 of s with tensor scale *g_out, in the prepared image
 * -- byte for byte what nvfp4_linear followed by nvfp4_swiglu_quantize with
 * g_in = g_out write, in one launch.
 * a_prepared, g_a: the M-row activation (as nvfp4_linear), 1 <= M <= 16.
 * w_prepared, g_w: nvfp4_prepare_weight of the [2F, K] gate+up weight (gate
 *   rows first); F % 128 == 0, K % 64 == 0.
 * g_out: device fp32, the static scale of the SwiGLU output (pass it as g_a
 *   of the down linear).  act_out: nvfp4_prepared_act_bytes(F) bytes;
 *   rows m < M are written.
 * ws: nvfp4_linear_swiglu_workspace_bytes(M, F, K) bytes, zero-filled at
 *   allocation and again after a failing device status (the workspace rule).
 * Dynamic activation scales need a grid-wide amax of s: use nvfp4_linear and
 * nvfp4_swiglu_quantize instead.
 * ---------------------------------------------------------------------- */
NVFP4SK_API size_t nvfp4_linear_swiglu_workspace_bytes(int64_t M, int64_t F, int64_t K);
NVFP4SK_API nvfp4sk_status nvfp4_linear_swiglu(const uint8_t *a_prepared, const float *g_a, int64_t M,
                                               const uint8_t *w_prepared, const float *g_w, int64_t F, int64_t K,
                                               const float *g_out, uint8_t *act_out, void *ws, size_t ws_bytes,
                                               nvfp4sk_stream_t stream);

/* ------------------------------------------------------------------------
 * nvfp4_linear_wide -- the same NVFP4 linear for many tokens at once: the
 * linears of the suffix prefill (section "KV-cache reuse between agent
 * steps": after the reused prefix is restored only the new suffix of the
 * prompt is prefilled, hundreds of tokens in one forward pass).
 * Y[s][n] = bf16( g_a*g_w * sum_b s_a[s,b] s_w[n,b] sum_{k in b} a[s,k] w[n,k]
 * (+ residual[s][n]) ), fp32 accumulation, for s < S.
 *
 * a_prepared: the S x K activation in the weight tile image, i.e. what
 *   nvfp4_prepare_weight(codes, scales, S, K, ...) writes for its canonical
 *   NVFP4 codes and scales (tokens take the place of weight rows);
 *   nvfp4_prepared_weight_bytes(S, K) bytes.  g_a: its tensor scale.
 * w_prepared, g_w: as nvfp4_linear.  S >= 1, N >= 1, K % 64 == 0.
 * residual: NULL or bf16 [S][ldy] added before rounding (may alias y).
 * y: bf16 [S][ldy], ldy >= N.  No workspace: every output tile is computed
 * whole by one CTA (tiles of 128 weight rows x 256 tokens).
 * ---------------------------------------------------------------------- */
NVFP4SK_API nvfp4sk_status nvfp4_linear_wide(const uint8_t *a_prepared, const float *g_a, int64_t S,
                                             const uint8_t *w_prepared, const float *g_w, int64_t N, int64_t K,
                                             const void *residual, void *y, int64_t ldy, nvfp4sk_stream_t stream);

/* ------------------------------------------------------------------------
 * nvfp4_linear_noalloc -- nvfp4_linear for callers that cannot allocate.
 * (The pages have no counterpart: this is a deployment variant.)
 *
 * Some callers cannot call cudaMalloc or take memory from a caching
 * allocator: a plugin inside a host runtime that owns all device memory, a
 * serving loop that must never enter an allocator on its latency path, or
 * code with no allocator at hand.  This variant takes no workspace: its
 * split-K scratch is a fixed array inside the library (every GPU that loads
 * the library holds nvfp4_linear_noalloc_scratch_bytes() of it until the
 * process exits).  Same arguments and results as nvfp4_linear otherwise.
 * Limits: N <= 524288 (larger N is rejected with
 * NVFP4SK_ERR_UNSUPPORTED_SHAPE); the grid is capped at 160 CTAs.
 * The first call on a device looks up the array's device address (and sets
 * kernel attributes); make that first call before any stream capture.
 * All calls on a device share the one array, and each call clears its
 * arrival counters first: calls whose GPU work can overlap (unordered
 * streams) race on it and must not be issued.
 * ---------------------------------------------------------------------- */
NVFP4SK_API size_t nvfp4_linear_noalloc_scratch_bytes(void);
NVFP4SK_API nvfp4sk_status nvfp4_linear_noalloc(const uint8_t *a_prepared, const float *g_a, int64_t M,
                                                const uint8_t *w_prepared, const float *g_w, int64_t N, int64_t K,
                                                const void *residual, void *y, int64_t ldy,
                                                nvfp4sk_stream_t stream);

/* ------------------------------------------------------------------------
 * tree_attn_fp8kv -- attention of the T tree nodes over the FP8 paged KV
 * cache with the ancestor mask (section "Tree multi-token prediction": the
 * target model verifies all candidates of the tree in one forward pass;
 * section "NVFP4 and FP8": FP8 KV cache).
 *
 * q: bf16, node i head hq at q[i*ld_q + hq*D + d] (ld_q >= Hq*D, even).
 * Cache (one layer): k_pool u8 [n_pool_pages][Hkv][page_size][D]
 *   (token-major pages); v_pool u8 [n_pool_pages][Hkv][D*page_size], each
 *   (page, head) plane cut into tiles of 8 dimensions x 16 slots (128
 *   bytes): dimension d, slot t at byte ((d/8)*(page_size/16) + t/16)*128 +
 *   (d%8)*16 + t%16 of the plane.  Position p lives in page page_table[p /
 *   page_size], slot p % page_size.  Context positions are 0..ctx_len-1; the
 *   tree nodes' own K/V are at ctx_len + i (node i).
 * page_table: i32 [ceil((ctx_len+T)/page_size)] physical page ids.
 * parent: i32 [T], parent[0] == -1, 0 <= parent[i] < i (topological order).
 * k_scale, v_scale: fp32 [Hkv]; K = value(code) * k_scale[h] (same for V).
 * Node i, head hq (KV head h = hq / (Hq/Hkv)) attends to every context
 *   position and to the tree positions of {i} and its ancestors:
 *   out = softmax_p(sm_scale * q . K_p) . V_p, bf16 [T][Hq][D] (dense).
 * Slots of the last page past position ctx_len+T-1 may hold any bytes
 *   (NaN codes included); they do not reach the output.  A page id outside
 *   [0, n_pool_pages) skips that page (its positions get no weight) and is
 *   flagged NVFP4SK_ERR_OUT_OF_RANGE in the device status, as is a parent id
 *   outside [-1, T).
 * Supported: D == 128, page_size == 64, 1 <= T <= 16, Hq/Hkv <= 8.
 * act_prepared (nullable): the bf16 output rows are also NVFP4-quantised with
 *   the static tensor scale *g_act into the prepared activation image that
 *   nvfp4_linear reads (K = Hq*D, row i = node i), exactly as
 *   nvfp4_quantize_act(out, g_in = g_act) would; g_act must then be non-NULL.
 * ws: tree_attn_workspace_bytes(...) bytes, zero-filled at allocation (it
 *   starts with the per-head arrival counters of the fused combine; see the
 *   workspace rule above).
 * Ordering: with programmatic dependent launch on (NVFP4SK_OPT_PDL, the
 *   default), the kernel reads page_table and starts loading context pages
 *   (positions < ctx_len) before the preceding kernel on the stream has
 *   finished, as nvfp4_linear does with its weights.  No kernel that may
 *   still run when this one starts may write them: the immediately preceding
 *   kernel, and, when that kernel lets its dependents start before it waits
 *   on its own predecessor (nvfp4_linear and the static-scale quantisers do),
 *   that predecessor in turn.  kv_append_fp8 waits first, so "append, then
 *   attention" is safe.  Everything else (q, parent, the scales, the tree
 *   slots) is read after the preceding kernel has finished.
 * ---------------------------------------------------------------------- */
NVFP4SK_API size_t tree_attn_workspace_bytes(int T, int Hq, int Hkv, int D, int page_size, int64_t ctx_len);
NVFP4SK_API nvfp4sk_status tree_attn_fp8kv(const void *q, int64_t ld_q, int T, int Hq, int Hkv, int D,
                               const uint8_t *k_pool, const uint8_t *v_pool, int64_t n_pool_pages,
                               int page_size, const int32_t *page_table, int64_t ctx_len,
                               const int32_t *parent, const float *k_scale, const float *v_scale,
                               float sm_scale, void *out, const float *g_act, uint8_t *act_prepared,
                               void *ws, size_t ws_bytes, nvfp4sk_stream_t stream);

/* ------------------------------------------------------------------------
 * causal_attn_fp8kv -- the attention of the suffix prefill (section "KV-cache
 * reuse between agent steps": the new suffix of the prompt is prefilled
 * after the reused prefix pages are restored): T <= 128 new tokens at
 * positions ctx_len .. ctx_len+T-1, whose K/V are already in the cache
 * (kv_append_fp8), attend causally: token i, head hq sees every position up
 * to ctx_len + i.  Same layouts, scales and output as tree_attn_fp8kv with a
 * chain (parent[i] = i-1), computed 128 queries of one query head per CTA
 * (grid: splits x Hq), so each K/V page is read once per 128 queries.
 * Longer suffixes are cut into blocks of up to 128 tokens, block b at
 * ctx_len = start + 128 b.  Hq % Hkv == 0, Hq <= 64; D == 128,
 * page_size == 64.  No NVFP4 output.
 * ws: causal_attn_workspace_bytes(...) bytes, zero-filled at allocation
 *   (arrival counters at its start, as for tree_attn_fp8kv).
 * Ordering with programmatic dependent launch: as tree_attn_fp8kv (context
 *   pages before the preceding kernel finishes, the T new positions after).
 * ---------------------------------------------------------------------- */
NVFP4SK_API size_t causal_attn_workspace_bytes(int T, int Hq, int Hkv, int D, int page_size, int64_t ctx_len);
NVFP4SK_API nvfp4sk_status causal_attn_fp8kv(const void *q, int64_t ld_q, int T, int Hq, int Hkv, int D,
                                             const uint8_t *k_pool, const uint8_t *v_pool, int64_t n_pool_pages,
                                             int page_size, const int32_t *page_table, int64_t ctx_len,
                                             const float *k_scale, const float *v_scale, float sm_scale, void *out,
                                             void *ws, size_t ws_bytes, nvfp4sk_stream_t stream);

/* Conversion of V pages written token-major (plane = [page_size slots][D]
 * bytes, the same layout as the K pool) into the tiled plane layout that
 * tree_attn_fp8kv reads (see above), for caches filled elsewhere.  n_planes
 * (page, head) planes of D*page_size bytes each, contiguous in both buffers;
 * plane i of v_tiled receives plane i of v_token_major.  The bytes are only
 * moved (no arithmetic).  D % 8 == 0, page_size % 16 == 0, D*page_size <=
 * 16384, buffers 16-byte aligned and not overlapping. */
NVFP4SK_API nvfp4sk_status kv_v_pages_to_tiled(const uint8_t *v_token_major, uint8_t *v_tiled, int64_t n_planes,
                                               int D, int page_size, nvfp4sk_stream_t stream);

/* ------------------------------------------------------------------------
 * kv_page_restore -- restore cached KV pages of a reused prompt prefix into
 * the live page pool (section "KV-cache reuse between agent steps": the
 * runtime restores the cached attention KV pages; ~96% of prompt tokens
 * came from the hot cache).  dst page dst_ids[i] <- src page src_ids[i],
 * page_bytes each, i = 0..n-1, as one gather-copy kernel.
 * src_ids, dst_ids: device i32 [n]; ids outside [0, n_src_pages) /
 * [0, n_dst_pages) are skipped and flagged (NVFP4SK_ERR_OUT_OF_RANGE in the
 * device status).  page_bytes % 16 == 0, pools 16-byte aligned.  dst ids
 * should be distinct (duplicates race).
 * ---------------------------------------------------------------------- */
NVFP4SK_API nvfp4sk_status kv_page_restore(const uint8_t *src_pool, const int32_t *src_ids, uint8_t *dst_pool,
                               const int32_t *dst_ids, int64_t n, int64_t page_bytes, int64_t n_src_pages,
                               int64_t n_dst_pages, nvfp4sk_stream_t stream);

/* ------------------------------------------------------------------------
 * Layer glue of the 64-layer verify step (not on the pages; fused where the
 * next op is an NVFP4 linear so that activations are quantised in the same
 * kernel that produces them).
 * ---------------------------------------------------------------------- */
/* y = x / sqrt(mean(x^2) + eps) * w rounded to bf16, then NVFP4-quantised
 * exactly as nvfp4_quantize_act, with the same outputs: g_in NULL = dynamic
 * tensor scale (amax over the whole y), else the static scale *g_in (a
 * calibrated checkpoint's; one launch with no grid-wide reduction).  x bf16
 * [rows][n] (row stride n), w bf16 [n].  rows <= 16, n % 64 == 0, n <= 8192;
 * with a static g_in and only the canonical outputs (act_prepared NULL) any
 * number of rows (the suffix prefill).  With a static g_in and programmatic
 * dependent launch on, w is read before the preceding kernel on the stream
 * has finished, as nvfp4_linear reads its weights: no kernel that may still
 * run may write it (see tree_attn_fp8kv for the rule). */
NVFP4SK_API nvfp4sk_status nvfp4_rmsnorm_quantize(const void *x, const void *w, float eps, int64_t rows,
                                                  int64_t n, const float *g_in, uint8_t *codes, uint8_t *scales,
                                                  float *g_out, uint8_t *act_prepared, void *ws, size_t ws_bytes,
                                                  nvfp4sk_stream_t stream);
/* h = silu(gu[:, :F]) * gu[:, F:] rounded to bf16, then NVFP4-quantised
 * (g_in NULL = dynamic g, else static *g_in), same outputs.  gu bf16
 * [rows][2F].  rows <= 16, F % 64 == 0, rows * F <= 524288; with a static
 * g_in and only the canonical outputs any number of rows. */
NVFP4SK_API nvfp4sk_status nvfp4_swiglu_quantize(const void *gu, int64_t rows, int64_t F, const float *g_in,
                                                 uint8_t *codes, uint8_t *scales, float *g_out, uint8_t *act_prepared,
                                                 void *ws, size_t ws_bytes, nvfp4sk_stream_t stream);
/* The static-scale quantisers of nvfp4_quantize_act, nvfp4_rmsnorm_quantize
 * and nvfp4_swiglu_quantize writing, instead of the canonical codes and
 * scales, the tile image that nvfp4_linear_wide streams for a many-token
 * activation: byte for byte what nvfp4_prepare_weight(codes, scales, rows, K)
 * writes for their canonical outputs, in one launch (the suffix prefill's
 * quantisation sites).  g_in: the static tensor scale (required); g_out
 * receives it.  tiles: nvfp4_prepared_weight_bytes(rows, K) bytes, 16-byte
 * aligned; the bytes of rows past `rows` in the last 128-row tile are not
 * written (only those tokens' outputs read them).  K (n, F) % 512 == 0;
 * rows >= 1; nvfp4_rmsnorm_quantize_tiles needs n <= 8192 and reads w before
 * the preceding kernel has finished, as nvfp4_rmsnorm_quantize does. */
NVFP4SK_API nvfp4sk_status nvfp4_quantize_act_tiles(const void *x, int x_dtype, int64_t rows, int64_t K,
                                                    int64_t ld_x, const float *g_in, float *g_out, uint8_t *tiles,
                                                    nvfp4sk_stream_t stream);
NVFP4SK_API nvfp4sk_status nvfp4_rmsnorm_quantize_tiles(const void *x, const void *w, float eps, int64_t rows,
                                                        int64_t n, const float *g_in, float *g_out, uint8_t *tiles,
                                                        nvfp4sk_stream_t stream);
NVFP4SK_API nvfp4sk_status nvfp4_swiglu_quantize_tiles(const void *gu, int64_t rows, int64_t F, const float *g_in,
                                                       float *g_out, uint8_t *tiles, nvfp4sk_stream_t stream);
/* Append T new tokens' K and V (bf16, token i head h at k_new[i*ld_new +
 * h*D + d]) to the cache at positions ctx_len .. ctx_len+T-1 as
 * E4M3(fp32(x / scale[h])) (round-to-nearest-even, saturating); the FP8 KV
 * cache write of section "NVFP4 and FP8".  Layouts as tree_attn_fp8kv;
 * D % 8 == 0 and page_size % 16 == 0. */
NVFP4SK_API nvfp4sk_status kv_append_fp8(const void *k_new, const void *v_new, int64_t ld_new, int T, int Hkv, int D,
                             uint8_t *k_pool, uint8_t *v_pool, int64_t n_pool_pages, int page_size,
                             const int32_t *page_table, int64_t ctx_len, const float *k_scale,
                             const float *v_scale, nvfp4sk_stream_t stream);
/* ------------------------------------------------------------------------
 * Greedy acceptance of the verified tree (section "Tree multi-token
 * prediction": all candidates are checked by one target pass and the path
 * that agrees with the target is kept; with greedy decoding that is exact).
 * Node 0 (the root, the last accepted token) is accepted; node i >= 1 is
 * accepted when its parent is accepted and draft_tokens[i] ==
 * target_argmax[parent[i]] (target_argmax[j]: the target's greedy token after
 * node j, e.g. from argmax_rows_bf16 of the LM head).  path (device i32 [T])
 * receives the node indices from the root to the deepest accepted node (lowest
 * index among equally deep ones), n_accepted (device i32 [1]) its length,
 * next_token (device i32 [1]) the target's token after that node.  parent
 * must be topologically ordered (parent[0] == -1, 0 <= parent[i] < i); else
 * only the root is accepted and NVFP4SK_ERR_OUT_OF_RANGE is flagged in the
 * device status.  1 <= T <= 32.
 * ---------------------------------------------------------------------- */
NVFP4SK_API nvfp4sk_status tree_accept_greedy(const int32_t *draft_tokens, const int32_t *target_argmax,
                                              const int32_t *parent, int T, int32_t *path, int32_t *n_accepted,
                                              int32_t *next_token, nvfp4sk_stream_t stream);
/* Move the accepted tokens' K/V next to the context in every layer: for k <
 * *n_accepted, the K and V bytes of logical position ctx_len + path[k] go to
 * position ctx_len + k (all are read before any is written).  Pools as
 * tree_attn_fp8kv; layer l's pools start at k_pool + l*layer_stride and
 * v_pool + l*layer_stride (bytes).  path / n_accepted as written by
 * tree_accept_greedy (device memory, so the two calls need no host sync).
 * Ids outside the pool or the tree are skipped and flagged
 * NVFP4SK_ERR_OUT_OF_RANGE.  D <= 128, D % 8 == 0, page_size % 16 == 0. */
NVFP4SK_API nvfp4sk_status kv_compact_accepted(uint8_t *k_pool, uint8_t *v_pool, int64_t layer_stride, int n_layers,
                                               int Hkv, int D, int64_t n_pool_pages, int page_size,
                                               const int32_t *page_table, int64_t ctx_len, const int32_t *path,
                                               const int32_t *n_accepted, int T, nvfp4sk_stream_t stream);
/* idx[r] = argmax_j x[r*ld + j] over bf16 values, lowest index on ties. */
NVFP4SK_API size_t argmax_workspace_bytes(int64_t rows, int64_t n);
NVFP4SK_API nvfp4sk_status argmax_rows_bf16(const void *x, int64_t rows, int64_t n, int64_t ld, int32_t *idx, void *ws,
                                size_t ws_bytes, nvfp4sk_stream_t stream);

/* ------------------------------------------------------------------------
 * Status, options, diagnostics
 * ---------------------------------------------------------------------- */
/* Synchronises `stream`, then reads and clears the device error word.
 * Returns NVFP4SK_OK, NVFP4SK_ERR_TIMEOUT or NVFP4SK_ERR_OUT_OF_RANGE;
 * *site (if non-NULL) receives the id of the last failing check. */
NVFP4SK_API nvfp4sk_status nvfp4sk_get_device_status(nvfp4sk_stream_t stream, int *site);
NVFP4SK_API const char *nvfp4sk_last_error(void);
NVFP4SK_API int nvfp4sk_version(void);

enum {
    NVFP4SK_OPT_PDL = 0,          /* 1: launch with programmatic dependent launch (default 1) */
    NVFP4SK_OPT_TIMEOUT_NS = 1,   /* per-wait limit of device spin-waits (default 1e9)        */
    NVFP4SK_OPT_ATTN_SPLITS = 2,  /* 0: automatic; else KV splits per KV head                 */
    NVFP4SK_OPT_LINEAR_CTAS = 3,  /* 0: one CTA per SM; else the split-K grid size            */
    NVFP4SK_OPT_ATTN_FUSED_COMBINE = 4 /* 1: the attention's CTAs merge their split results
                                        themselves (needs splits x heads <= #SMs); 0 (default):
                                        a second launch merges them (measured faster on B200) */
};
NVFP4SK_API nvfp4sk_status nvfp4sk_set_option(int option, int64_t value);
NVFP4SK_API int64_t nvfp4sk_get_option(int option);

/* Diagnostic: element-wise device conversion of fp32 values with the same
 * instructions the quantisers use: e2m1[i] = E2M1 code (low nibble), e4m3[i]
 * = E4M3 code (RNE, satfinite).  Either output may be NULL. */
NVFP4SK_API nvfp4sk_status nvfp4sk_debug_encode(const float *x, int64_t n, uint8_t *e2m1, uint8_t *e4m3,
                                    nvfp4sk_stream_t stream);

/* Diagnostic (failure detection; the pages have no counterpart): one launch
 * whose single device wait can never be satisfied.  The wait gives up after
 * the NVFP4SK_OPT_TIMEOUT_NS limit; the next nvfp4sk_get_device_status
 * returns NVFP4SK_ERR_TIMEOUT with site 900, and the context stays usable. */
NVFP4SK_API nvfp4sk_status nvfp4sk_debug_wait_timeout(nvfp4sk_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* NVFP4SK_H */
