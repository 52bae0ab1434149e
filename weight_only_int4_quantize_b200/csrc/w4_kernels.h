// Internal launcher declarations of libw4 (host side).  The public C ABI is
// include/w4.h; these functions assume already-validated arguments.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace w4 {

constexpr int kMaxGrid = 64;  // alphas / shrinks per scoring call

struct AlphaList {
  int n;
  float v[kMaxGrid];
};
struct ShrinkList {
  int n;
  float v[kMaxGrid];
};

// Up to kQuantBatch tensors quantized by one launch (kernel parameter).
constexpr int kQuantBatch = 64;
struct QuantBatch {
  int count;
  const void* w[kQuantBatch];
  const float* s[kQuantBatch];
  float shrink[kQuantBatch];
  const float* shrink_rows[kQuantBatch];  // per-row ratios [N] (device) or NULL
  void* qw[kQuantBatch];
  uint16_t* scales[kQuantBatch];
  uint16_t* zeros[kQuantBatch];
  int64_t n_groups[kQuantBatch];
  int64_t groups_per_row[kQuantBatch];
  int64_t unit_start[kQuantBatch + 1];  // prefix sums of ceil(groups / 32) (chunks)
};
void quant_batch_add(QuantBatch& b, const void* w, int64_t N, int64_t K, const float* s,
                     float shrink, int32_t* qweight, uint16_t* scales, uint16_t* zeros,
                     const float* shrink_rows = nullptr);
cudaError_t launch_quantize_pack_batch(const QuantBatch& b, bool symmetric, cudaStream_t stream,
                                       int num_sms, unsigned* err);

// Up to kGemvBatch independent linears with the same token count (<= 16)
// decoded by one launch; tensor maps travel in the kernel parameter.
constexpr int kGemvBatch = 32;
struct GemvBatch {
  CUtensorMap tw[kGemvBatch];  // packed codes, uint8 [N, K/2], box 64 x 64
  CUtensorMap tx[kGemvBatch];  // x, bf16 [M, K], box 64 x tokens, 128B swizzle
  const __nv_bfloat16* xp[kGemvBatch];  // x, bf16 [M, K] (read directly for <= 8 tokens)
  const uint16_t* scales[kGemvBatch];
  const uint16_t* zeros[kGemvBatch];
  __nv_bfloat16* y[kGemvBatch];
  int N[kGemvBatch];
  int K[kGemvBatch];
  int cta_start[kGemvBatch + 1];  // prefix sums of 64-row blocks
  int count, M, ksplit, gs_max;
};
cudaError_t gemv_batch_add(GemvBatch& b, const void* x, const int32_t* qw, const uint16_t* sc,
                           const uint16_t* z, int N, int K, void* y);
cudaError_t launch_gemv_batch(GemvBatch& b, bool symmetric, bool pdl, bool static_w,
                              cudaStream_t stream, int num_sms, unsigned* err);
cudaError_t launch_gemv(const void* x, int M, const int32_t* qw, const uint16_t* sc,
                        const uint16_t* z, int N, int K, void* y, bool pdl, bool static_w,
                        cudaStream_t stream, int num_sms, unsigned* err);

// Up to kStreamBatch independent linears with the same token count (<= 8)
// decoded by one persistent streaming launch (kernel parameter).
constexpr int kStreamBatch = 256;
struct StreamBatch {
  const __nv_bfloat16* x[kStreamBatch];  // bf16 [M, K]; W4A8: int8 codes [M, K]
  const uint8_t* qw[kStreamBatch];       // packed codes, [N, K/2] bytes
  const uint16_t* scales[kStreamBatch];  // fp16 [N, K/128]
  const uint16_t* zeros[kStreamBatch];   // fp16 [N, K/128]; NULL: symmetric
  __nv_bfloat16* y[kStreamBatch];        // bf16 [M, N]
  int N[kStreamBatch];
  int K[kStreamBatch];
  const int32_t* xsum[kStreamBatch];     // W4A8: per-group code sums [M, K/128]
  const float* xscale[kStreamBatch];     // W4A8: per-token scales [M]
  int ks[kStreamBatch];                  // K parts of each linear (1, 2 or 4)
  int unit_start[kStreamBatch + 1];      // prefix sums of bundles (4 warp units each)
  int count, M;
  int a8;                                // activations: 0 bf16, 1 int8 codes
};
void stream_batch_add(StreamBatch& b, const void* x, const int32_t* qw, const uint16_t* sc,
                      const uint16_t* z, int N, int K, void* y, const int32_t* xsum = nullptr,
                      const float* xscale = nullptr);
// Chooses the K split of every linear for the launch's grid; *bundles is the
// number of 4-warp bundles the launch would deal (launch_gemv_stream plans
// the same way, so planning first does not change the launch).
cudaError_t plan_gemv_stream(StreamBatch& b, bool symmetric, int num_sms, int* bundles);
cudaError_t launch_gemv_stream(StreamBatch& b, bool symmetric, bool pdl, bool static_w,
                               cudaStream_t stream, int num_sms);

// One linear of a grouped prefill launch (all share M).
struct PrefillItem {
  const void* x;       // bf16 [M, K]
  const int32_t* qw;   // packed [N, K/8]
  const uint16_t* sc;  // fp16 [N, K/128]
  const uint16_t* z;   // fp16 [N, K/128]; NULL: symmetric (the same for all items)
  void* y;             // bf16 [M, N]
  int N, K;
};
// Tile shape (rows x cols) and K split (CTAs per cluster) of a prefill launch.
struct PrefillPlan {
  int rows, cols, ks;
};
// Tile shapes in the order of the `resident` tables: 256 x 256, 128 x 256,
// 256 x 128, 128 x 128; K splits 1 .. 4.
constexpr int kPrefillShapes = 4;
constexpr int kPrefillMaxSplit = 4;
// CTAs of each tile shape that the current device runs at once in clusters
// of 1 .. 4 (asked of the runtime once per device; estimated while `stream`
// is being captured and the counts are not known yet).
void prefill_resident(int sms, cudaStream_t stream,
                      int (&resident)[kPrefillShapes][kPrefillMaxSplit]);
// The plan of one grouped launch of n <= 16 linears (N[i] x K[i], sharing M
// rows) from the launch's time model; host arithmetic only.
PrefillPlan plan_prefill_group(const int* N, const int* K, int n, int M,
                               const int (&resident)[kPrefillShapes][kPrefillMaxSplit]);
// Up to 16 linears per tcgen05 launch (more in further launches).
cudaError_t launch_prefill_gemm_group(const PrefillItem* items, int count, int M, bool pdl,
                                      bool static_w, cudaStream_t stream, unsigned* err);
// Per-token int8 activation codes (channel order 0,4,1,5,2,6,3,7 in every
// 8-channel chunk), per-group code sums and per-token scales.
cudaError_t launch_quantize_act_int8(const void* x, int64_t M, int64_t K, int8_t* xq,
                                     int32_t* xsum, float* xscale, cudaStream_t stream);

cudaError_t launch_prefill_gemm(const void* x, int M, const int32_t* qw, const uint16_t* sc,
                                const uint16_t* z, int N, int K, void* y, bool pdl,
                                bool static_w, cudaStream_t stream, unsigned* err);

cudaError_t launch_sumsq_gemm(const void* a_f16, int M, const void* b_f16, int N, int K,
                              int n_cand, double* partials, int n_seg, const int* seg_off,
                              cudaStream_t stream, unsigned* err);
int sumsq_tiles(int M, int N);
// Per-column sums of (A . B_c^T)^2 over the rows of each row tile:
// partials[c][row_tile][n] in binary64 (fixed order).
cudaError_t launch_colsumsq_gemm(const void* a_f16, int M, const void* b_f16, int N, int K,
                                 int n_cand, double* partials, cudaStream_t stream,
                                 unsigned* err);
int colsumsq_row_tiles(int M);

cudaError_t launch_awq_scales(const void* x, int64_t M, int64_t K, const AlphaList& alphas,
                              float* s_out, cudaStream_t stream);
// Operand exponents (awq.cu): partial column maxima of |x| and |w| over
// colmax_chunks(R) row chunks, then per alpha fe[2i] = f_i, fe[2i+1] = e_i.
int colmax_chunks(int64_t R);
cudaError_t launch_colmax_abs(const void* a, int64_t R, int64_t K, float* part,
                              cudaStream_t stream);
cudaError_t launch_awq_exponents(const float* xpart, int xchunks, const float* wpart, int wchunks,
                                 const float* s_all, int n_alpha, int64_t K, int* fe,
                                 cudaStream_t stream);
cudaError_t launch_awq_xs(const void* x, const float* s, int64_t M, int64_t K, const int* fexp,
                          void* a, cudaStream_t stream, int num_sms);
cudaError_t launch_awq_err(const void* w, const float* s, int64_t N, int64_t K, bool symmetric,
                           const ShrinkList& shrinks, const int* eexp, void* e,
                           cudaStream_t stream, int num_sms);
cudaError_t launch_awq_reduce(const double* partials, int n_cand, int n_seg, int tiles, int n_r,
                              const int* fe, double* sse, cudaStream_t stream);
cudaError_t launch_awq_argmin(const double* sse, int n_seg, int n_a, int n_r, int c1,
                              int32_t* out, cudaStream_t stream);

cudaError_t launch_clip_rows_select(const double* partials, int n_cand, int row_tiles, int64_t N,
                                    const ShrinkList& shrinks, const int* fe, double* sse_rows,
                                    int32_t* choice, float* shrink_rows, cudaStream_t stream);
cudaError_t launch_fill_ones(float* p, int64_t n, cudaStream_t stream);

// Exact (binary64) decision of near ties (awq.cu).  At most kExactCap
// candidates of an awq_score_grid call are decided again.
constexpr int kExactCap = 64;
struct SegOffsets {
  int off[17];
};
cudaError_t launch_exact_rowsse(const void* x, int M, const void* w, int N, int K,
                                const float* s_all, const ShrinkList& shrinks, int n_r,
                                bool symmetric, const int* list, const int* count, int cap,
                                const int* rowlist, const int* rowcount, const uint32_t* cmask,
                                const SegOffsets& seg, int n_seg, double* rowsum,
                                cudaStream_t stream);
cudaError_t launch_awq_flag(const double* sse, int n_seg, int n_a, int n_r, int c1, double tol,
                            int cap, int* list, int* count, uint32_t* masks, cudaStream_t stream);
// Token chunks of the binary64 kernel: its row sums are [cap][chunks][N].
int exact_token_chunks(int M);
cudaError_t launch_awq_exact_merge(const double* rowsum, int M, int N, const int* list,
                                   const int* count, const uint32_t* masks, int cap, int n_seg,
                                   const SegOffsets& seg, int n_c, double* sse,
                                   cudaStream_t stream);
cudaError_t launch_clip_exact(const void* x, int M, const void* w, int N, int K, const float* s,
                              const ShrinkList& shrinks, bool symmetric, double tol,
                              double* sse_rows, int32_t* choice, float* shrink_rows,
                              uint8_t* flags, unsigned long long* mask, int* list, int* count,
                              int* rows, int* row_counts, double* rowsum, cudaStream_t stream);

// C[M, N] (pitch ldc, binary64) = r1 (+ r2) + 2^-(*ea + *eb) * A B^T with A
// fp16 [M, K] and B fp16 [N, K] row-major (K a multiple of 64), on the
// tcgen05 tensor cores with TMA-fed operands (gemm_tc.cu).
cudaError_t launch_add_gemm_f16(const void* a_f16, int M, const void* b_f16, int N, int K,
                                double* out, int ldc, const double* r1, const double* r2,
                                const int* ea, const int* eb, cudaStream_t stream,
                                unsigned* err);

// Block-level candidate scoring in binary64 (block.cu).  Linears in the
// order q, k, v, o, gate, up, down (bf16 [out, in]); groups 0 qkv, 1 o,
// 2 gate_up, 3 down.
struct BlockConfig {
  int hidden, heads, kv_heads, head_dim, ffn;
  double eps, rope_theta;
};
struct BlockNorms {
  const double* ln1;
  const double* ln2;
  const double* q_norm;
  const double* k_norm;
};
struct BlockLinears {
  const void* w[7];
  BlockNorms norms;
};
size_t block_workspace_bytes(const BlockConfig& c, int64_t T);
cudaError_t block_scoring_losses(const BlockConfig* c, const double* x, int64_t T,
                                 const BlockLinears& blk, const BlockLinears* next, int group,
                                 const float* alphas, int n_alpha, const float* shrinks,
                                 int n_shrink, bool sym, int only, double* losses,
                                 void* workspace, cudaStream_t st);
cudaError_t block_search(const BlockConfig* c, const double* x, int64_t T, const BlockLinears& blk,
                         const BlockLinears* next, const float* alphas, int n_alpha,
                         const float* shrinks, int n_shrink, bool sym, int32_t* choice,
                         double* losses, void* workspace, cudaStream_t st, unsigned* err);

// Device address of the fixed scratch behind awq_score_grid_static_scratch
// on the current device (looked up once per device, then cached).
cudaError_t awq_static_scratch_address(void** ptr);


}  // namespace w4
