// Internal launcher declarations of libw4 (host side).  The public C ABI is
// include/w4.h; these functions assume already-validated arguments.
#pragma once

#include <cstdint>
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

cudaError_t launch_quantize_pack(const void* w, int64_t N, int64_t K, bool symmetric,
                                 const float* s, float shrink, int32_t* qweight, uint16_t* scales,
                                 uint16_t* zeros, cudaStream_t stream, int num_sms);

cudaError_t launch_gemv(const void* x, int M, const int32_t* qw, const uint16_t* sc,
                        const uint16_t* z, int N, int K, void* y, bool pdl, bool static_w,
                        cudaStream_t stream, int num_sms, unsigned* err);

cudaError_t launch_prefill_gemm(const void* x, int M, const int32_t* qw, const uint16_t* sc,
                                const uint16_t* z, int N, int K, void* y, bool pdl,
                                bool static_w, cudaStream_t stream, unsigned* err);

cudaError_t launch_sumsq_gemm(const void* a_f16, int M, const void* b_f16, int N, int K,
                              int n_cand, double* partials, int n_seg, const int* seg_off,
                              cudaStream_t stream, unsigned* err);
int sumsq_tiles(int M, int N);

cudaError_t launch_awq_scales(const void* x, int64_t M, int64_t K, const AlphaList& alphas,
                              float* s_out, cudaStream_t stream);
cudaError_t launch_awq_xs(const void* x, const float* s, int64_t M, int64_t K, void* a,
                          cudaStream_t stream, int num_sms);
cudaError_t launch_awq_err(const void* w, const float* s, int64_t N, int64_t K, bool symmetric,
                           const ShrinkList& shrinks, void* e, cudaStream_t stream, int num_sms);
cudaError_t launch_awq_reduce(const double* partials, int n_cand, int n_seg, int tiles,
                              double* sse, cudaStream_t stream);
cudaError_t launch_awq_argmin(const double* sse, int n_seg, int n_a, int n_r, int c1,
                              int32_t* out, cudaStream_t stream);


}  // namespace w4
