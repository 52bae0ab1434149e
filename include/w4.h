/*
 * w4.h -- C ABI of libw4: weight-only int4 group-128 quantization, the W4A16
 * linear that consumes it (decode and prefill), the W4A8 decode over the
 * same stored weights, AWQ alpha/shrink candidate scoring and the
 * per-output-channel clipping search, the block-level (look-ahead) candidate
 * loss and search, as hand-written CUDA kernels for B200 (sm_100a).
 *
 * Sources (model-card pages, cited by title and section):
 *   [rebuttal] "ghostchoir/rebuttal_w4g128_awq_w2": 'Model Details' table
 *              rows 'Scheme' (weight-only, 4-bit, group size 128, asymmetric
 *              zero point) and 'Search' (AWQ scale exponent on a 20-point
 *              grid, clipping as a 10-point global shrink grid); the
 *              scale-rewrite paragraph (prev_op /= s, W *= s equals
 *              Q(W diag(s)) diag(1/s)); 'Clipping granularity' (one shrink
 *              ratio per linear); the table note defining RTN; the
 *              'Comparability caveat' (stock per-output-channel clipping).
 *   [qwen27b]  "GotoAI-Inc/Qwen3.6-27B-W4A16": opening paragraph (int4, group
 *              size 128, symmetric, weight-only, activations stay 16-bit).
 *   [awq-ppl]  "AWQ INT4-g128 WikiText-2 perplexity delta vs fp16, Llama-2
 *              7B": 'Methodology' (grid size 20 for the alpha search).
 *   [qsrt]     "malaiwah/GLM-5.2-QSRT-Fruit-Instruct": 'Reproducible runtime'
 *              (decode-sized batches of at most 16 rows take a separate
 *              path from prefill, W4A8 there); 'What is included' and the
 *              storage paragraph (W4A8 decode over the same stored weights).
 *   [q326]     "ariacompute/qwen3-1.7b_q326_channel": the Qwen3-1.7B block
 *              shapes used by the block-level scoring.
 *
 * Conventions shared by every entry point
 *   - Device pointers are caller-owned device memory (any allocator).  Host
 *     pointers are marked "host".  The library never allocates or frees
 *     memory and keeps no state between calls apart from one device-side
 *     error word (see w4_device_error).  The one fixed device array it holds,
 *     the scratch of awq_score_grid_static_scratch, carries nothing from one
 *     call to the next.
 *   - `stream` is a cudaStream_t passed as void*; NULL is the legacy default
 *     stream.  Launches are asynchronous; outputs are valid once the stream
 *     has been synchronized.
 *   - Arguments are validated on the host before anything is launched.  A
 *     call that returns anything but W4_OK has launched nothing.
 *   - Every device base pointer must be 16-byte aligned (per-row shrink
 *     ratios: 4-byte), unless an entry point states otherwise.
 *   - bf16 / fp16 buffers are passed as raw 16-bit patterns (void* /
 *     uint16_t*).  Inputs must be finite.
 *   - No C++ exception crosses the ABI; CUDA failures return W4_ERR_CUDA.
 *
 * Packed weight format (canonical; the pages give storage sizes only)
 *   qweight : int32 [N, K/8].  Word w of row n holds the eight 4-bit codes of
 *             input channels 8w..8w+7; nibble i (bits 4i..4i+3) holds channel
 *             8w + {0,2,4,6,1,3,5,7}[i], so nibbles (i, i+4) are the adjacent
 *             channels (2i, 2i+1).
 *   scales  : fp16 bits [N, K/128], row-major.
 *   zeros   : fp16 bits [N, K/128] holding integers 0..15 (asymmetric), or
 *             absent (symmetric: implicit zero 8).
 *   Dequantization: w_hat[n,k] = (q[n,k] - zero[n,k/128]) * scale[n,k/128].
 *   Storage: 0.53125 byte/weight asymmetric, 0.515625 symmetric.
 */
#ifndef W4_H
#define W4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  W4_OK = 0,
  W4_ERR_INVALID_ARG = 1,    /* NULL pointer where one is required, bad flag */
  W4_ERR_SHAPE = 2,          /* non-positive size, K not a multiple of 128, ... */
  W4_ERR_ALIGNMENT = 3,      /* a device pointer not 16-byte aligned */
  W4_ERR_UNSUPPORTED = 4,    /* group != 128, grid larger than supported, ... */
  W4_ERR_WORKSPACE = 5,      /* workspace missing or smaller than required */
  W4_ERR_CUDA = 6,           /* a CUDA runtime call failed (launch, attribute, ...) */
  W4_ERR_DEVICE_TIMEOUT = 7  /* a kernel gave up on a bounded wait (w4_device_error) */
} w4_status;

/* Static, NUL-terminated description of a status code. */
const char* w4_status_string(w4_status status);

/* Description of the last W4_ERR_CUDA returned on the calling host thread
 * (the failing step and the CUDA error name); empty if none.  Static storage
 * of the library, valid until the next call on that thread. */
const char* w4_last_error(void);

/* ABI version of this header (bumped on any incompatible change). */
#define W4_ABI_VERSION 1
int w4_abi_version(void);

/*
 * w4_quantize_pack -- round-to-nearest int4 group-128 quantization and
 * packing of one linear's weight ([rebuttal] 'Scheme'; [qwen27b]).
 *
 * w_bf16    device, bf16 [N, K] row-major (K contiguous): the weight W.
 * N, K      output and input features; N >= 1, K >= 128, K % 128 == 0.
 * group     must be 128.
 * symmetric 0: asymmetric with zero point; 1: symmetric.
 * awq_s     device, float32 [K], or NULL.  When given, the weight quantized
 *           is v = W * diag(s) (per input channel, binary32 multiply),
 *           i.e. the Q(W diag(s)) of [rebuttal]'s scale-rewrite paragraph.
 *           The caller folds 1/s into the op that produces x.
 * shrink    clipping shrink ratio r in (0, 1] ([rebuttal] 'Clipping
 *           granularity'); 1.0 is no clipping.
 * qweight   device, int32 [N, K/8] out.
 * scales_f16 device, fp16 bits [N, K/128] out.
 * zeros_f16 device, fp16 bits [N, K/128] out; must be NULL iff symmetric.
 *
 * Per group G of 128 consecutive channels of one row, in IEEE binary32 with
 * round-to-nearest-even and no fused multiply-add:
 *   asymmetric: mx = r*max v, mn = r*min v,
 *               scale = fp16_rn(max(mx - mn, 1e-5) / 15),
 *               zero  = clamp(rint(-mn / scale), 0, 15);
 *   symmetric:  scale = fp16_rn(max(r*max|v|, 1e-5) / 7), zero = 8;
 *   code = clamp(rint(v / scale) + zero, 0, 15)   (scale = the stored fp16
 *          value, rint ties to even, v/scale correctly rounded).
 * Bit-exact with the CPU oracle.  Returns W4_OK or a validation / CUDA error.
 */
w4_status w4_quantize_pack(const void* w_bf16, int64_t N, int64_t K, int group,
                           int symmetric, const float* awq_s, float shrink,
                           int32_t* qweight, uint16_t* scales_f16, uint16_t* zeros_f16,
                           void* stream);

/*
 * w4_quantize_pack_batched -- w4_quantize_pack over `count` independent
 * tensors (for example every linear of a model) in as few launches as
 * possible (64 tensors per launch).  Each item is validated as
 * w4_quantize_pack validates its arguments; `symmetric` and `group` apply to
 * all items; each item has its own optional AWQ scale and shrink ratio.
 * items: host array.  Results are bit-identical to per-tensor calls.
 */
typedef struct {
  const void* w_bf16;     /* device, bf16 [N, K] */
  int64_t N, K;
  const float* awq_s;     /* device, float32 [K], or NULL */
  float shrink;           /* (0, 1] */
  int32_t* qweight;       /* device, int32 [N, K/8] out */
  uint16_t* scales_f16;   /* device, fp16 [N, K/128] out */
  uint16_t* zeros_f16;    /* device, fp16 [N, K/128] out; NULL iff symmetric */
} w4_quant_item;
w4_status w4_quantize_pack_batched(const w4_quant_item* items, int count, int group,
                                   int symmetric, void* stream);

/*
 * w4a16_linear -- y = x . dequant(Wq)^T with bf16 activations and a bf16
 * result ([qwen27b]: activations stay 16-bit; [qsrt] 'Reproducible runtime':
 * decode-sized row counts take their own path).  No bias.
 *
 * x_bf16    device, bf16 [M, K] row-major.
 * M         token rows, 1 <= M <= 2^31-1.
 * qweight, scales_f16, zeros_f16  the packed weight (zeros NULL: symmetric).
 * N, K      as for w4_quantize_pack.
 * group     must be 128.
 * y_bf16    device, bf16 [M, N] row-major out (accumulated in binary32,
 *           rounded once to bf16).
 * flags     bitwise OR of W4_LINEAR_* below (0 for defaults).
 *
 * M <= 32 (and K <= 81920) runs a decode GEMV (tensor-core mma over
 * register-dequantized weight fragments, HBM-bound); larger M runs the
 * prefill GEMM (tcgen05 with TMEM accumulators, weight tiles dequantized into
 * shared memory).  There are two decode kernels: a persistent streaming
 * kernel (M <= 8; every warp streams 64-row units through its own ring) for
 * launches with at least two of its 4-warp bundles per SM, and a per-CTA
 * tensor-map kernel (K split over a thread-block cluster) for smaller
 * launches and 9 <= M <= 64.  W4_LINEAR_DECODE_STREAM / _TILED override the
 * choice; both meet the same error bound.  A prefill launch picks its tile
 * shape (128 or 256 rows x 128 or 256 columns) and a split of K over a
 * thread-block cluster of up to 4 CTAs from a time model measured on B200 and
 * the number of CTAs the device runs at once in clusters of each size (asked
 * of the runtime once per device; a launch captured into a graph before any
 * uncaptured one on its device estimates it).  The fp32 partial tiles are
 * added through distributed shared memory in rank order, so a given launch
 * configuration always gives the same bits.
 */
#define W4_LINEAR_FORCE_GEMV 0x1u  /* decode kernel at any M <= 64 (K <= 81920) */
#define W4_LINEAR_FORCE_GEMM 0x2u  /* prefill kernel at any M */
#define W4_LINEAR_PDL 0x4u         /* programmatic dependent launch: the
                                      kernel may start before the previous
                                      kernel on the stream ends and waits for
                                      it before touching global memory */
#define W4_LINEAR_STATIC_WEIGHTS 0x8u /* with W4_LINEAR_PDL: the caller
                                      guarantees qweight/scales/zeros are not
                                      written by preceding work still in
                                      flight, so the kernel may start streaming
                                      them before the dependency wait */
#define W4_LINEAR_DECODE_STREAM 0x10u /* decode through the persistent
                                      streaming kernel (M <= 8 only) */
#define W4_LINEAR_DECODE_TILED 0x20u  /* decode through the per-CTA
                                      tensor-map kernel (M <= 64) */
w4_status w4a16_linear(const void* x_bf16, int64_t M, const int32_t* qweight,
                       const uint16_t* scales_f16, const uint16_t* zeros_f16,
                       int64_t N, int64_t K, int group, void* y_bf16,
                       unsigned flags, void* stream);

/*
 * w4a16_linear_batched -- w4a16_linear over `count` independent linears that
 * share the token count M and the symmetry (all zeros NULL or none), for
 * example every projection of a decode step whose inputs are ready.  M <= 8
 * runs up to 256 linears per persistent streaming launch (or, for a launch
 * too small to fill the GPU, the tensor-map kernel); 9 <= M <= 32 (K <=
 * 81920) runs the tensor-map kernel with up to 32 linears per launch (up to
 * M = 64 with W4_LINEAR_DECODE_TILED); larger M runs grouped prefill GEMM
 * launches, up to 16 linears each (every CTA finds its linear and tile; the
 * tile shape and K split are chosen for the group).  flags: W4_LINEAR_PDL,
 * W4_LINEAR_STATIC_WEIGHTS and the W4_LINEAR_DECODE_* choice only.  items: host array.  Each result meets the
 * same error bound as a per-linear call (the K split of a batch, and so the
 * binary32 summation order, may differ from a single call's).
 */
typedef struct {
  const void* x_bf16;          /* device, bf16 [M, K] */
  const int32_t* qweight;      /* device, packed weight */
  const uint16_t* scales_f16;
  const uint16_t* zeros_f16;   /* NULL: symmetric */
  int64_t N, K;
  void* y_bf16;                /* device, bf16 [M, N] out */
} w4_linear_item;
w4_status w4a16_linear_batched(const w4_linear_item* items, int count, int64_t M, int group,
                               unsigned flags, void* stream);

/*
 * w4_prefill_plan -- the tile shape and K split that a prefill launch uses
 * (w4a16_linear above 32 rows, or one launch of w4a16_linear_batched) for
 * `count` linears of N[i] x K[i] weights that share the token count M.  For
 * inspection and tuning: it computes the launch's own choice (the time model
 * described at w4a16_linear) and launches nothing.
 *
 * N, K       host int64 [count]; N >= 1, K a positive multiple of 128.
 * count      1 .. 16 (a launch takes at most 16 linears).
 * M          >= 1.
 * resident   NULL: the current device's counts (asks the runtime); else host
 *            int [16]: for the tile shapes 256 x 256, 128 x 256, 256 x 128 and
 *            128 x 128 (rows x columns) in that order, the CTAs that run at
 *            once in clusters of 1, 2, 3 and 4 CTAs (each >= 1).  With
 *            resident given no device is used.
 * tile_rows, tile_cols, k_split  host int out: the CTA tile and the number
 *            of CTAs that split K in a cluster (1: no split).
 * Returns W4_ERR_INVALID_ARG (NULL pointer, count out of range, a resident
 * count < 1) or W4_ERR_SHAPE; with resident NULL, W4_ERR_CUDA without a
 * usable device.
 */
w4_status w4_prefill_plan(const int64_t* N, const int64_t* K, int count, int64_t M,
                          const int* resident, int* tile_rows, int* tile_cols, int* k_split);

/*
 * W4A8 decode -- the same stored int4 weights against int8 activations
 * ([qsrt] 'What is included': W4A8 decode execution; the storage paragraph:
 * W4A8 and W4A16 use the same stored weights; the runtime paragraph: W4A8
 * for decode-sized batches of at most 16 rows).  The pages fix no
 * activation format; this library quantizes per token, symmetric:
 *
 *   xscale[m] = max_k |x_mk| / 127               (binary32)
 *   xq[m, k]  = clamp(rint(x_mk / xscale[m]), -127, 127)
 *               (IEEE division, ties to even; a zero row has scale 0, codes 0)
 *   xsum[m, g] = sum_{k in group g} xq[m, k]      (int32)
 *   y[m, n] = xscale[m] * sum_g scale[n, g] * sum_{k in g} (q[n, k] - z[n, g]) * xq[m, k]
 *
 * The group sums are exact integers (int8 x int4 tensor-core products with
 * int32 accumulation); the scaling and the sum over groups run in binary32
 * and y is rounded once to bf16.
 *
 * w4_quantize_act_int8 -- x_bf16 device bf16 [M, K] (K % 128 == 0) ->
 *   xq_out int8 [M, K] (in every 8-channel chunk the channels are stored in
 *   the order 0, 4, 1, 5, 2, 6, 3, 7, the order in which the nibble masks of
 *   a packed weight word deliver its codes), xsum_out int32 [M, K/128],
 *   xscale_out float32 [M].  All device, 16-byte aligned.  One quantization
 *   serves every linear that reads the same x (q, k, v; gate, up).
 * w4a8_linear -- y_bf16 [M, N] from those three arrays and a packed weight
 *   (as for w4a16_linear), 1 <= M <= 16, K <= 81920; flags W4_LINEAR_PDL and
 *   W4_LINEAR_STATIC_WEIGHTS only.  Runs the persistent streaming decode
 *   kernel (8 tokens per launch).
 * w4a8_linear_batched -- many such linears (host array of w4a8_item) sharing
 *   M and the symmetry, up to 256 per launch.
 */
w4_status w4_quantize_act_int8(const void* x_bf16, int64_t M, int64_t K, int8_t* xq_out,
                               int32_t* xsum_out, float* xscale_out, void* stream);
w4_status w4a8_linear(const int8_t* xq, const int32_t* xsum, const float* xscale, int64_t M,
                      const int32_t* qweight, const uint16_t* scales_f16,
                      const uint16_t* zeros_f16, int64_t N, int64_t K, int group, void* y_bf16,
                      unsigned flags, void* stream);
typedef struct {
  const int8_t* xq;            /* device, int8 [M, K] (w4_quantize_act_int8 layout) */
  const int32_t* xsum;         /* device, int32 [M, K/128] */
  const float* xscale;         /* device, float32 [M] */
  const int32_t* qweight;      /* device, packed weight */
  const uint16_t* scales_f16;
  const uint16_t* zeros_f16;   /* NULL: symmetric */
  int64_t N, K;
  void* y_bf16;                /* device, bf16 [M, N] out */
} w4a8_item;
w4_status w4a8_linear_batched(const w4a8_item* items, int count, int64_t M, int group,
                              unsigned flags, void* stream);

/*
 * w4_awq_scales -- AWQ per-input-channel scales ([rebuttal] 'Search': AWQ
 * scale exponent grid; [awq-ppl] 'Methodology': grid of 20 alphas).
 *
 *   stat_j = (sum_m |x_mj|) / M   (binary64, fixed summation order m = 0..M-1)
 *   s[i, j] = (float) pow(max(stat_j, 1e-8), alpha_i)   (binary64 pow)
 *
 * x_bf16   device, bf16 [M, K];  M >= 1, K >= 1.
 * alphas   host, float32 [n_alpha], 1 <= n_alpha <= 64.
 * s_out    device, float32 [n_alpha, K] out.
 */
w4_status w4_awq_scales(const void* x_bf16, int64_t M, int64_t K, const float* alphas,
                        int n_alpha, float* s_out, void* stream);

/*
 * awq_score_grid -- batched AWQ candidate scoring over the alpha x shrink
 * grid ([rebuttal] 'Search' and the scale-rewrite paragraph: a candidate is
 * simulated by swapping only the linear's weight for
 * Q(W diag(s)) diag(1/s)).  For every (alpha_i, shrink_j):
 *
 *   s = w4_awq_scales(x, alpha_i),  What = dequant(Q_r(W diag(s))) diag(1/s),
 *   SSE[seg, i, j] = || x . (W - What)^T ||_F^2 over the rows of W in seg.
 *
 * The candidate's codes are bit-identical to w4_quantize_pack(W, s, shrink).
 * The error product runs on tcgen05 tensor cores in fp16 in the s-domain,
 * (x/s) . (W s - w_hat)^T, each operand scaled by an exact power of two
 * chosen from its column maxima (its largest values near the top of fp16's
 * range), accumulated in binary32, squared and summed in binary64 with the
 * scaling removed exactly.  Every selection of argmin_out whose fp16 values
 * put two or more candidates within 5e-4 (relative) of its least value is
 * decided again on values recomputed from scratch in binary64 (fp64 MMA)
 * for those candidates (at most 64 per call), whose sse_out entries are then
 * the binary64 values: the selections are those of the binary64 definition,
 * up to the order of its sums.
 *
 * x_bf16       device, bf16 [M, K] calibration activations.
 * w_bf16       device, bf16 [N, K] weight of one linear, or of several
 *              linears that share x concatenated along N (q,k,v; gate,up).
 * group        must be 128;  symmetric as for w4_quantize_pack.
 * alphas       host, float32 [n_alpha], 1 <= n_alpha <= 64.
 * shrinks      host, float32 [n_shrink], 1 <= n_shrink <= 64, each in (0,1].
 * seg_offsets  host, int64 [n_seg + 1] with 0 = off[0] < ... < off[n_seg] = N,
 *              interior offsets multiples of 16; or NULL with n_seg = 1.
 * n_seg        1..16 linears sharing x.
 * sse_out      device, float64 [n_seg, n_alpha, n_shrink] out.
 * argmin_out   device, int32 [n_seg + 1, 4] out.  Row s < n_seg:
 *              {joint flat argmin (alpha-major), alpha* at shrink 1.0,
 *               shrink* at that alpha*, shrink* at the group's alpha*};
 *              row n_seg: {joint argmin of the summed table, the group's
 *              alpha* (summed table at shrink 1.0), -1, -1}.  "Shrink 1.0" is
 *              the first shrink equal to 1.0f, else column 0.  Equal minima
 *              resolve to the lowest index.
 * workspace    device scratch of at least w4_awq_workspace_bytes(...) bytes,
 *              256-byte aligned; contents on entry are ignored.
 */
size_t w4_awq_workspace_bytes(int64_t M, int64_t N, int64_t K, int n_alpha, int n_shrink,
                              int n_seg);
w4_status awq_score_grid(const void* x_bf16, int64_t M, const void* w_bf16, int64_t N,
                         int64_t K, int group, int symmetric, const float* alphas,
                         int n_alpha, const float* shrinks, int n_shrink,
                         const int64_t* seg_offsets, int n_seg, double* sse_out,
                         int32_t* argmin_out, void* workspace, size_t workspace_bytes,
                         void* stream);

/*
 * awq_score_grid_static_scratch -- awq_score_grid without a caller-supplied
 * workspace: its scratch is a fixed device array inside the library of
 * W4_AWQ_STATIC_SCRATCH_BYTES (32 MiB).  The pages have no counterpart.  The
 * candidates, SSE table and argmins are those of awq_score_grid,
 * bit-identical for the same inputs (every reduction runs in a fixed order).
 *
 * It is for callers that cannot allocate device memory when they score: a
 * serving process whose caching allocator already holds the free HBM (for
 * weights and KV cache), so that a fresh cudaMalloc of the workspace fails;
 * and a caller in the middle of queued asynchronous work, where cudaFree's
 * implicit device-wide synchronization would stall the pipeline.  The call
 * allocates nothing (no cudaMalloc, cudaFree or allocating library routine).
 *
 * Size limit: a problem whose w4_awq_workspace_bytes(M, N, K, n_alpha,
 * n_shrink, n_seg) exceeds W4_AWQ_STATIC_SCRATCH_BYTES is refused with
 * W4_ERR_WORKSPACE, nothing launched; w4_last_error() then names the needed
 * and available sizes.  Any other invalid argument returns the same status
 * as awq_score_grid would, checked before anything else (the scratch is
 * not looked up then).
 *
 * Set-up: the first call on each device, with that device current, looks up
 * the scratch's device address (cudaGetSymbolAddress) and caches it; under
 * CUDA's default lazy module loading this is also when the driver reserves
 * the 32 MiB on that device.  Make that first call before any stream capture
 * begins.  The cached address (like the device error word's, see
 * w4_device_error) belongs to the device's primary context: do not use the
 * library across cudaDeviceReset or another teardown of that context.
 *
 * Nothing in the scratch needs to start at zero: every word a kernel of the
 * call reads is written earlier in the same call, so nothing is cleared.
 *
 * Concurrency: there is one scratch per device.  Calls whose work overlaps on
 * one device (different streams, or several host threads) race on it and
 * produce undefined results; order them on one stream.
 *
 * Arguments as for awq_score_grid, without workspace and workspace_bytes.
 */
#define W4_AWQ_STATIC_SCRATCH_BYTES (32u << 20)
w4_status awq_score_grid_static_scratch(const void* x_bf16, int64_t M, const void* w_bf16,
                                        int64_t N, int64_t K, int group, int symmetric,
                                        const float* alphas, int n_alpha,
                                        const float* shrinks, int n_shrink,
                                        const int64_t* seg_offsets, int n_seg,
                                        double* sse_out, int32_t* argmin_out, void* stream);

/*
 * awq_clip_search_rows -- stock per-output-channel clipping search
 * ([rebuttal] 'Comparability caveat': the d=0 arm clips with stock AWQ's
 * per-output-channel search; 'Clipping granularity' contrasts it with the one
 * global ratio a look-ahead loss forces).  For one AWQ scale s (or none) and
 * a grid of shrink ratios r_j, every output row n takes the ratio whose
 * quantization error has the least output error in that row:
 *
 *   E_j = W - dequant(Q_{r_j}(W diag(s))) diag(1/s)
 *   sse_rows[j, n] = sum_m (x E_j^T)[m, n]^2        (binary64, fixed order)
 *   choice[n] = argmin_j sse_rows[j, n]              (lowest j on equal values)
 *
 * The linear's output error is the sum of its rows' errors, so the choices
 * minimise it jointly over all per-row ratio assignments.  Scored in the
 * s-domain on fp16 tensor-core operands with binary64 sums, like
 * awq_score_grid (same codes as w4_quantize_pack); a row whose fp16 values
 * put two or more ratios within 5e-3 (relative) of its least value has
 * those ratios' errors recomputed in binary64 and chooses on them.
 *
 * x_bf16, M      device bf16 [M, K] calibration activations, 1 <= M <= 2^24.
 * w_bf16, N, K   device bf16 [N, K] weight, 1 <= N <= 2^24, K % 128 == 0.
 * group          must be 128.
 * symmetric      0: asymmetric with zero point; 1: symmetric.
 * awq_s          device float32 [K] AWQ scale (for instance one row of
 *                w4_awq_scales), or NULL for none (s = 1).
 * shrinks        host float32 [n_shrink], each in (0, 1]; 1 <= n_shrink <= 64.
 * sse_rows_out   device float64 [n_shrink, N] out.
 * choice_out     device int32 [N] out: index into shrinks.
 * shrink_rows_out  device float32 [N] out (the chosen ratios, ready for
 *                w4_quantize_pack_rows), or NULL.
 * workspace      device scratch of at least w4_clip_rows_workspace_bytes(...)
 *                bytes, 256-byte aligned.
 * Errors: as awq_score_grid.  Nothing is launched unless every check passes.
 */
size_t w4_clip_rows_workspace_bytes(int64_t M, int64_t N, int64_t K, int n_shrink);
w4_status awq_clip_search_rows(const void* x_bf16, int64_t M, const void* w_bf16, int64_t N,
                               int64_t K, int group, int symmetric, const float* awq_s,
                               const float* shrinks, int n_shrink, double* sse_rows_out,
                               int32_t* choice_out, float* shrink_rows_out, void* workspace,
                               size_t workspace_bytes, void* stream);

/*
 * Block-level candidate scoring (binary64 losses; the search screened on
 * tcgen05 tensor cores with binary64 decisions).
 *
 * [rebuttal] 'Model Details' table, row 'Search', and the paragraph under
 * it: a candidate (alpha, shrink) for a linear group of decoder block i is
 * scored by the mean squared difference, over tokens and hidden units,
 * between the output of block i+1 (kept in original precision) with the
 * candidate's quantized linears swapped into block i and the same path with
 * block i unquantized; block i's own output when there is no successor (the
 * last block, and the perplexity table's d=0 arm).  A candidate swaps only
 * its linears' weights for Q_r(W diag(s)) diag(1/s) (scale-rewrite
 * paragraph; the codes of w4_quantize_pack), s = fp32(max(stat, 1e-8)^alpha)
 * with stat the mean |input| over tokens of the activation entering the
 * group on the unquantized path.  Block shapes: [q326] "ariacompute/
 * qwen3-1.7b_q326_channel" (16 query heads, 8 key/value heads of width 128,
 * SwiGLU width 6144).  The decoder block follows the Qwen3 conventions (the
 * pages do not give it): pre-norm RMSNorm, per-head RMSNorm of q and k, then
 * a rotate-half rotary embedding at positions 0..T-1, causal softmax
 * attention scaled by 1/sqrt(head_dim), query head h reading key/value head
 * h / (heads / kv_heads), SwiGLU MLP (silu(gate) * up), residual adds.
 *
 * awq_block_scoring_losses runs every step in binary64 (the contractions on
 * the fp64 MMA); its results depend on nothing but the inputs (fixed order
 * of every sum).  awq_block_search screens first (see there).
 *
 * Linears are numbered q 0, k 1, v 2, o 3, gate 4, up 5, down 6; groups are
 * qkv 0 (q, k, v), o 1, gate_up 2 (gate, up), down 3.
 */
typedef struct {
  int32_t hidden;     /* multiple of 128 */
  int32_t heads;      /* query heads */
  int32_t kv_heads;   /* key/value heads, divides heads */
  int32_t head_dim;   /* 64 or 128; heads * head_dim a multiple of 128 */
  int32_t ffn;        /* SwiGLU width, multiple of 128 */
  double eps;         /* RMSNorm epsilon, > 0 */
  double rope_theta;  /* rotary base, > 0 */
} w4_block_config;

typedef struct {
  /* device bf16 [out, in] row-major: q [heads*head_dim, hidden], k and v
   * [kv_heads*head_dim, hidden], o [hidden, heads*head_dim], gate and up
   * [ffn, hidden], down [hidden, ffn] */
  const void* q;
  const void* k;
  const void* v;
  const void* o;
  const void* gate;
  const void* up;
  const void* down;
  const double* ln1;     /* device float64 [hidden]: the attention norm gain */
  const double* ln2;     /* device float64 [hidden]: the MLP norm gain */
  const double* q_norm;  /* device float64 [head_dim] */
  const double* k_norm;  /* device float64 [head_dim] */
} w4_block_weights;

/* Workspace of awq_block_scoring_losses and awq_block_search for T tokens:
 * six sets of block activations (each about (heads T^2 + 16 T max(hidden,
 * ffn)) * 8 bytes), the largest group's binary64 candidate weights and the
 * fp16 copies of both blocks' weights; 0 if cfg is NULL or T < 1. */
size_t w4_block_workspace_bytes(const w4_block_config* cfg, int64_t T);

/*
 * awq_block_scoring_losses -- loss[a, j] of every candidate (alphas[a],
 * shrinks[j]) of one linear group.  The shrink applies to every linear of
 * the group, or with only >= 0 to that linear alone (the group's other
 * linears quantized at the same alpha, unclipped).
 *
 * cfg            host, the block shape.
 * x, T           device float64 [T, hidden]: block i's input; 1 <= T <= 8192.
 * block          host struct of device pointers: block i.
 * next           host struct: block i+1 (loss at its output), or NULL (loss
 *                at block i's output).
 * group          0..3.   only: -1, or a linear of the group.
 * alphas         host float32 [n_alpha], finite; 1 <= n_alpha <= 64.
 * shrinks        host float32 [n_shrink], each in (0, 1]; 1 <= n_shrink <= 64.
 * symmetric      0: asymmetric with zero point; 1: symmetric.
 * losses_out     device float64 [n_alpha, n_shrink] out.
 * workspace      device scratch of at least w4_block_workspace_bytes(cfg, T)
 *                bytes, 256-byte aligned.
 * Errors: W4_ERR_INVALID_ARG (NULL pointer, group / only / grid value out of
 * range), W4_ERR_SHAPE (a size outside the ranges above),
 * W4_ERR_UNSUPPORTED (head_dim, grid sizes), W4_ERR_ALIGNMENT,
 * W4_ERR_WORKSPACE, W4_ERR_CUDA.  Nothing is launched unless every check
 * passes.  Stream-ordered; no host synchronization.
 */
w4_status awq_block_scoring_losses(const w4_block_config* cfg, const double* x, int64_t T,
                                   const w4_block_weights* block, const w4_block_weights* next,
                                   int group, const float* alphas, int n_alpha,
                                   const float* shrinks, int n_shrink, int symmetric, int only,
                                   double* losses_out, void* workspace, size_t workspace_bytes,
                                   void* stream);

/*
 * awq_block_search -- the search of one block ([rebuttal] 'Search' row,
 * 'Clipping granularity'): for each group in order, alpha* = the least loss
 * over the alpha grid at shrink 1 (every linear of the group quantized with
 * that alpha); then for each linear of the group its own ratio r* = the
 * least loss over the shrink grid with the group at alpha* and its other
 * linears unclipped.  Groups are scored one at a time with the rest of
 * block i unquantized.  Ties go to the lowest index.
 *
 * Every selection is screened first: the reference paths run once in
 * binary64 with their intermediates kept, and a candidate's path is the
 * reference plus its change, each linear's change a tcgen05 product of fp16
 * operands scaled by exact powers of two (attention, norms and SwiGLU in
 * binary64 on the full values).  The candidates whose screening loss is
 * within 1e-3 (relative) of the least are scored again on the binary64 path
 * of awq_block_scoring_losses, and the selection takes the least of those
 * binary64 losses: the choices are those of the binary64 definition.  The
 * call synchronizes the stream once per selection (the near-tie sets are
 * read on the host).
 *
 * choice_out     device int32 [11] out: alpha index per group (4), then
 *                shrink index per linear (7).
 * losses_out     device float64 [4 * n_alpha + 7 * n_shrink] out (the alpha
 *                losses per group, then the shrink losses per linear: the
 *                binary64 value for a candidate of a near-tie set, else its
 *                screening value), or NULL.
 * Other arguments and errors as awq_block_scoring_losses.
 */
w4_status awq_block_search(const w4_block_config* cfg, const double* x, int64_t T,
                           const w4_block_weights* block, const w4_block_weights* next,
                           const float* alphas, int n_alpha, const float* shrinks, int n_shrink,
                           int symmetric, int32_t* choice_out, double* losses_out,
                           void* workspace, size_t workspace_bytes, void* stream);

/*
 * w4_quantize_pack_rows -- w4_quantize_pack with one shrink ratio per output
 * row (the weight that per-output-channel clipping deploys, [rebuttal]
 * 'Comparability caveat').  shrink_rows: device float32 [N], 4-byte aligned,
 * each expected in (0, 1] (device data, not checked: a ratio outside that
 * range quantizes its row with that wider or degenerate range, and never
 * reads or writes out of bounds).  Every other argument, the layouts and the
 * arithmetic are those of w4_quantize_pack; a row's codes, scales and zeros
 * equal w4_quantize_pack of that row alone with its ratio.
 */
w4_status w4_quantize_pack_rows(const void* w_bf16, int64_t N, int64_t K, int group,
                                int symmetric, const float* awq_s, const float* shrink_rows,
                                int32_t* qweight, uint16_t* scales_f16, uint16_t* zeros_f16,
                                void* stream);

/*
 * w4_device_error -- reads (and with clear != 0 resets) the library's device
 * error word.  Every wait inside the tcgen05 kernels is bounded (about one
 * second); a kernel that gives up records it here and returns early, leaving
 * its outputs undefined but the CUDA context usable.  Synchronize the streams
 * that ran library kernels first.  Returns W4_OK, W4_ERR_DEVICE_TIMEOUT or
 * W4_ERR_CUDA; *code_out (may be NULL) receives the raw word (0 = none).
 */
w4_status w4_device_error(int clear, uint32_t* code_out);

/*
 * w4_selftest_bounded_wait -- launches one CTA that waits on a shared-memory
 * barrier nobody arrives at, with the given limit in nanoseconds
 * (1e6..2e9), then gives up, records the timeout in the device error word and
 * returns.  Exercises the failure path of the bounded waits without faulting
 * or hanging the GPU.
 */
w4_status w4_selftest_bounded_wait(uint64_t limit_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* W4_H */
