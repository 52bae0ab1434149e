// AWQ alpha x shrink candidate scoring ("ghostchoir/rebuttal_w4g128_awq_w2"
// model card, 'Model Details' row 'Search' and the scale-rewrite paragraph).
//
// For each alpha_i the scales s = max(mean_m |x_m|, 1e-8)^alpha_i are formed
// once; the candidate error of shrink r_j is scored in the s-domain,
//   x . (W - dequant(Q_r(W diag(s))) diag(1/s))^T
//     = (x diag(1/s)) . (W diag(s) - dequant(Q_r(W diag(s))))^T,
// with both tensor-core operands brought into fp16's normal range by exact
// powers of two chosen per alpha from the largest possible magnitudes:
//   A_i = fp16((x / s) * 2^f_i)          [M, K]   (awq_xs_kernel)
//   E_ij = fp16((w*s - w_hat) * 2^e_i)   [N, K]   (awq_err_kernel, all shrinks
//                                                  of one alpha in one pass)
// with f_i = 14 - floor(log2 max_k(max_m |x_mk| / s_k)) and
// e_i = 13 - floor(log2 max_k(max_n |w_nk| * s_k)), so |A| < 2^15 and
// |E| <= 2 max |w s| < 2^15; the squared sums are multiplied back by
// 4^-(f_i + e_i) (exact in binary64).
// The tcgen05 GEMM (gemm_tc.cu) squares and sums A_i . E_ij^T per tile in
// binary64; awq_reduce_kernel adds the tile sums in fixed order and
// awq_argmin_kernel takes the selections.  The codes of every candidate are
// the quantize+pack kernel's codes (same quant_group.cuh arithmetic).
//
// The per-output-channel clipping search ("Comparability caveat" of the same
// card: stock AWQ's per-output-channel clipping) uses the same operands for
// one s and the shrink grid, a per-column epilogue of the same GEMM, and
// clip_rows_select_kernel for each row's least-error ratio.
#include "quant_group.cuh"
#include "w4_kernels.h"

namespace w4 {

namespace {

// stat_j = sum_m |x_mj| / M in binary64 (m = 0..M-1 in order), then
// s[i, j] = (float) pow(max(stat_j, 1e-8), (double) alpha_i).
__global__ void awq_scales_kernel(const __nv_bfloat16* __restrict__ x, int64_t M, int64_t K,
                                  AlphaList alphas, float* __restrict__ s_out) {
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j >= K) return;
  double acc = 0.0;
  const unsigned short* xb = reinterpret_cast<const unsigned short*>(x);
  for (int64_t m = 0; m < M; ++m) {
    const float v = __uint_as_float(static_cast<uint32_t>(__ldg(xb + m * K + j)) << 16);
    acc += static_cast<double>(fabsf(v));
  }
  const double stat = fmax(acc / static_cast<double>(M), 1e-8);
  for (int i = 0; i < alphas.n; ++i) {
    const double a = static_cast<double>(alphas.v[i]);
    s_out[static_cast<int64_t>(i) * K + j] = static_cast<float>(pow(stat, a));
  }
}

// Partial column maxima of |a| over row chunks: part[c][k] = max over rows
// r = c, c + chunks, ... of |a[r, k]| (no atomics; reduced by the exponent
// kernel).
__global__ void colmax_abs_kernel(const __nv_bfloat16* __restrict__ a, int64_t R, int64_t K,
                                  float* __restrict__ part) {
  const int64_t k = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (k >= K) return;
  const unsigned short* ab = reinterpret_cast<const unsigned short*>(a);
  float mx = 0.f;
  for (int64_t r = blockIdx.y; r < R; r += gridDim.y)
    mx = fmaxf(mx, fabsf(__uint_as_float(static_cast<uint32_t>(__ldg(ab + r * K + k)) << 16)));
  part[static_cast<int64_t>(blockIdx.y) * K + k] = mx;
}

// Per alpha (one block each): fe[2i] = f_i, fe[2i + 1] = e_i (see the file
// comment); 0 when the corresponding maximum is 0.
__global__ void awq_exponents_kernel(const float* __restrict__ xpart, int xchunks,
                                     const float* __restrict__ wpart, int wchunks,
                                     const float* __restrict__ s_all, int64_t K,
                                     int* __restrict__ fe) {
  __shared__ float red[2][32];
  const float* s = s_all + static_cast<int64_t>(blockIdx.x) * K;
  float ma = 0.f, mw = 0.f;
  for (int64_t k = threadIdx.x; k < K; k += blockDim.x) {
    float xm = 0.f, wm = 0.f;
    for (int c = 0; c < xchunks; ++c) xm = fmaxf(xm, xpart[c * K + k]);
    for (int c = 0; c < wchunks; ++c) wm = fmaxf(wm, wpart[c * K + k]);
    ma = fmaxf(ma, __fdiv_rn(xm, s[k]));
    mw = fmaxf(mw, __fmul_rn(wm, s[k]));
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    ma = fmaxf(ma, __shfl_xor_sync(0xffffffffu, ma, o));
    mw = fmaxf(mw, __shfl_xor_sync(0xffffffffu, mw, o));
  }
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) {
    red[0][w] = ma;
    red[1][w] = mw;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 1; i < static_cast<int>(blockDim.x >> 5); ++i) {
      ma = fmaxf(ma, red[0][i]);
      mw = fmaxf(mw, red[1][i]);
    }
    fe[2 * blockIdx.x] = ma > 0.f ? 14 - ilogbf(ma) : 0;
    fe[2 * blockIdx.x + 1] = mw > 0.f ? 13 - ilogbf(mw) : 0;
  }
}

// A = fp16(fl(x / s) * 2^f): correctly rounded binary32 division, an exact
// power-of-two scaling, then fp16 RNE.
__global__ void awq_xs_kernel(const __nv_bfloat16* __restrict__ x, const float* __restrict__ s,
                              int64_t M, int64_t K, const int* __restrict__ fexp,
                              __half* __restrict__ a) {
  const int f = fexp ? __ldg(fexp) : 0;
  const int64_t n8 = M * K / 8;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint4 r = __ldg(reinterpret_cast<const uint4*>(x) + i);
    float v[8];
    bf16x8_to_f32(r, v);
    const int64_t k0 = (i * 8) % K;
    const float4 s0 = __ldg(reinterpret_cast<const float4*>(s + k0));
    const float4 s1 = __ldg(reinterpret_cast<const float4*>(s + k0 + 4));
    const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
    uint32_t o[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const __half2 h =
          __halves2half2(__float2half_rn(ldexpf(__fdiv_rn(v[2 * p], sv[2 * p]), f)),
                         __float2half_rn(ldexpf(__fdiv_rn(v[2 * p + 1], sv[2 * p + 1]), f)));
      o[p] = *reinterpret_cast<const uint32_t*>(&h);
    }
    reinterpret_cast<uint4*>(a)[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// E_j[n, k] = fp16((v - w_hat) * 2^e) with v = w*s and w_hat = (q - zero)*scale
// the candidate's exact dequantized value, for every shrink j, one half warp
// per 128-value group (same lane layout as the quantize kernel).
template <bool SYM>
__global__ void __launch_bounds__(256)
    awq_err_kernel(const uint4* __restrict__ w, const float* __restrict__ s, int64_t n_groups,
                   int64_t groups_per_row, ShrinkList shrinks, int64_t plane_elems,
                   const int* __restrict__ eexp, __half* __restrict__ e) {
  const int ex = eexp ? __ldg(eexp) : 0;
  const int lane = threadIdx.x & 31;
  const int half = lane >> 4;
  const int l16 = lane & 15;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x) >> 5;
  const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * 256) >> 5;
  const int64_t n_units = (n_groups + 1) >> 1;
  for (int64_t u = warp; u < n_units; u += n_warps) {
    const int64_t gi = 2 * u + half;
    const bool valid = gi < n_groups;
    const uint4 raw = valid ? __ldg(w + gi * 16 + l16) : make_uint4(0, 0, 0, 0);
    float v[8];
    bf16x8_to_f32(raw, v);
    const int64_t k0 = (gi % groups_per_row) * 128 + l16 * 8;
    if (valid) {
      const float4 s0 = __ldg(reinterpret_cast<const float4*>(s + k0));
      const float4 s1 = __ldg(reinterpret_cast<const float4*>(s + k0 + 4));
      v[0] = __fmul_rn(v[0], s0.x); v[1] = __fmul_rn(v[1], s0.y);
      v[2] = __fmul_rn(v[2], s0.z); v[3] = __fmul_rn(v[3], s0.w);
      v[4] = __fmul_rn(v[4], s1.x); v[5] = __fmul_rn(v[5], s1.y);
      v[6] = __fmul_rn(v[6], s1.z); v[7] = __fmul_rn(v[7], s1.w);
    }
    float gmax, gmin = 0.f;
    if (SYM) {
      float a = fabsf(v[0]);
#pragma unroll
      for (int j = 1; j < 8; ++j) a = fmaxf(a, fabsf(v[j]));
      gmax = hw_max(a);
    } else {
      float mx = v[0], mn = v[0];
#pragma unroll
      for (int j = 1; j < 8; ++j) { mx = fmaxf(mx, v[j]); mn = fminf(mn, v[j]); }
      gmax = hw_max(mx);
      gmin = hw_min(mn);
    }
    for (int r = 0; r < shrinks.n; ++r) {
      const GroupQ g = group_params<SYM>(gmax, gmin, shrinks.v[r]);
      uint32_t o[4];
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        float d[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float val = v[2 * p + h];
          const float q = static_cast<float>(code_of(val, g));
          const float what = __fmul_rn(__fsub_rn(q, g.zero), g.sc);  // exact
          d[h] = ldexpf(__fsub_rn(val, what), ex);
        }
        const __half2 h2 = __halves2half2(__float2half_rn(d[0]), __float2half_rn(d[1]));
        o[p] = *reinterpret_cast<const uint32_t*>(&h2);
      }
      if (valid)
        reinterpret_cast<uint4*>(e + r * plane_elems + gi * 128)[l16] =
            make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

// SSE[seg, i, j] = 4^-(f_i + e_i) * sum over tiles (fixed order) of the
// GEMM's tile sums.
__global__ void awq_reduce_kernel(const double* __restrict__ partials, int n_cand, int n_seg,
                                  int tiles, int n_r, const int* __restrict__ fe,
                                  double* __restrict__ sse) {
  const int id = blockIdx.x * blockDim.x + threadIdx.x;  // = seg * n_cand + cand
  if (id >= n_cand * n_seg) return;
  const int seg = id / n_cand;
  const int cand = id % n_cand;
  const double* p = partials + (static_cast<size_t>(cand) * n_seg + seg) * tiles;
  double sum = 0.0;
  for (int t = 0; t < tiles; ++t) sum += p[t];
  const int i = cand / n_r;
  sse[id] = ldexp(sum, -2 * (fe[2 * i] + fe[2 * i + 1]));
}

// Selections, lowest index on equal values (single thread; <= 64x64 tables).
__global__ void awq_argmin_kernel(const double* __restrict__ sse, int n_seg, int n_a, int n_r,
                                  int c1, int32_t* __restrict__ out) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  auto at = [&](int s, int i, int j) { return sse[(static_cast<size_t>(s) * n_a + i) * n_r + j]; };
  auto total = [&](int i, int j) {
    double t = 0.0;
    for (int s = 0; s < n_seg; ++s) t += at(s, i, j);
    return t;
  };
  int a_grp = 0;
  for (int i = 1; i < n_a; ++i)
    if (total(i, c1) < total(a_grp, c1)) a_grp = i;
  for (int s = 0; s < n_seg; ++s) {
    int joint = 0;
    for (int f = 1; f < n_a * n_r; ++f)
      if (at(s, f / n_r, f % n_r) < at(s, joint / n_r, joint % n_r)) joint = f;
    int a_s = 0;
    for (int i = 1; i < n_a; ++i)
      if (at(s, i, c1) < at(s, a_s, c1)) a_s = i;
    int r_s = 0, r_g = 0;
    for (int j = 1; j < n_r; ++j) {
      if (at(s, a_s, j) < at(s, a_s, r_s)) r_s = j;
      if (at(s, a_grp, j) < at(s, a_grp, r_g)) r_g = j;
    }
    out[4 * s + 0] = joint;
    out[4 * s + 1] = a_s;
    out[4 * s + 2] = r_s;
    out[4 * s + 3] = r_g;
  }
  int joint = 0;
  for (int f = 1; f < n_a * n_r; ++f)
    if (total(f / n_r, f % n_r) < total(joint / n_r, joint % n_r)) joint = f;
  out[4 * n_seg + 0] = joint;
  out[4 * n_seg + 1] = a_grp;
  out[4 * n_seg + 2] = -1;
  out[4 * n_seg + 3] = -1;
}

// Per-output-channel clipping: sse_rows[c, n] = sum over row tiles (fixed
// order) of the column sums, choice[n] = the lowest c of least error, and
// the chosen ratio itself.  One thread per output channel.
__global__ void clip_rows_select_kernel(const double* __restrict__ partials, int n_cand,
                                        int row_tiles, int64_t N, ShrinkList shrinks,
                                        const int* __restrict__ fe,
                                        double* __restrict__ sse_rows, int32_t* __restrict__ choice,
                                        float* __restrict__ shrink_rows) {
  const int64_t n = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (n >= N) return;
  const int sc = -2 * (fe[0] + fe[1]);
  int best = 0;
  double best_v = 0.0;
  for (int c = 0; c < n_cand; ++c) {
    double v = 0.0;
    for (int t = 0; t < row_tiles; ++t) v += partials[(static_cast<size_t>(c) * row_tiles + t) * N + n];
    v = ldexp(v, sc);
    sse_rows[static_cast<size_t>(c) * N + n] = v;
    if (c == 0 || v < best_v) {
      best = c;
      best_v = v;
    }
  }
  choice[n] = best;
  if (shrink_rows) shrink_rows[n] = shrinks.v[best];
}

__global__ void fill_ones_kernel(float* __restrict__ p, int64_t n) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    p[i] = 1.0f;
}

}  // namespace

cudaError_t launch_clip_rows_select(const double* partials, int n_cand, int row_tiles, int64_t N,
                                    const ShrinkList& shrinks, const int* fe, double* sse_rows,
                                    int32_t* choice, float* shrink_rows, cudaStream_t stream) {
  const int64_t blocks = (N + 127) / 128;
  clip_rows_select_kernel<<<static_cast<unsigned>(blocks), 128, 0, stream>>>(
      partials, n_cand, row_tiles, N, shrinks, fe, sse_rows, choice, shrink_rows);
  return cudaGetLastError();
}

int colmax_chunks(int64_t R) { return R < 32 ? static_cast<int>(R) : 32; }

cudaError_t launch_colmax_abs(const void* a, int64_t R, int64_t K, float* part,
                              cudaStream_t stream) {
  const dim3 grid(static_cast<unsigned>((K + 127) / 128), static_cast<unsigned>(colmax_chunks(R)));
  colmax_abs_kernel<<<grid, 128, 0, stream>>>(static_cast<const __nv_bfloat16*>(a), R, K, part);
  return cudaGetLastError();
}

cudaError_t launch_awq_exponents(const float* xpart, int xchunks, const float* wpart, int wchunks,
                                 const float* s_all, int n_alpha, int64_t K, int* fe,
                                 cudaStream_t stream) {
  awq_exponents_kernel<<<n_alpha, 256, 0, stream>>>(xpart, xchunks, wpart, wchunks, s_all, K, fe);
  return cudaGetLastError();
}

cudaError_t launch_fill_ones(float* p, int64_t n, cudaStream_t stream) {
  fill_ones_kernel<<<static_cast<unsigned>((n + 255) / 256 < 1024 ? (n + 255) / 256 : 1024), 256,
                     0, stream>>>(p, n);
  return cudaGetLastError();
}

cudaError_t launch_awq_scales(const void* x, int64_t M, int64_t K, const AlphaList& alphas,
                              float* s_out, cudaStream_t stream) {
  const int threads = 128;
  const int64_t blocks = (K + threads - 1) / threads;
  awq_scales_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(x), M, K, alphas, s_out);
  return cudaGetLastError();
}

cudaError_t launch_awq_xs(const void* x, const float* s, int64_t M, int64_t K, const int* fexp,
                          void* a, cudaStream_t stream, int num_sms) {
  const int64_t n8 = M * K / 8;
  int64_t blocks = (n8 + 255) / 256;
  if (blocks > static_cast<int64_t>(num_sms) * 8) blocks = static_cast<int64_t>(num_sms) * 8;
  awq_xs_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(x), s, M, K, fexp, static_cast<__half*>(a));
  return cudaGetLastError();
}

cudaError_t launch_awq_err(const void* w, const float* s, int64_t N, int64_t K, bool symmetric,
                           const ShrinkList& shrinks, const int* eexp, void* e,
                           cudaStream_t stream, int num_sms) {
  const int64_t n_groups = N * (K / 128);
  const int64_t n_units = (n_groups + 1) / 2;
  int64_t blocks = (n_units + 7) / 8;
  if (blocks > static_cast<int64_t>(num_sms) * 8) blocks = static_cast<int64_t>(num_sms) * 8;
  const uint4* wp = static_cast<const uint4*>(w);
  __half* ep = static_cast<__half*>(e);
  if (symmetric)
    awq_err_kernel<true><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        wp, s, n_groups, K / 128, shrinks, N * K, eexp, ep);
  else
    awq_err_kernel<false><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        wp, s, n_groups, K / 128, shrinks, N * K, eexp, ep);
  return cudaGetLastError();
}

cudaError_t launch_awq_reduce(const double* partials, int n_cand, int n_seg, int tiles, int n_r,
                              const int* fe, double* sse, cudaStream_t stream) {
  const int n = n_cand * n_seg;
  awq_reduce_kernel<<<(n + 127) / 128, 128, 0, stream>>>(partials, n_cand, n_seg, tiles, n_r, fe,
                                                         sse);
  return cudaGetLastError();
}

cudaError_t launch_awq_argmin(const double* sse, int n_seg, int n_a, int n_r, int c1,
                              int32_t* out, cudaStream_t stream) {
  awq_argmin_kernel<<<1, 32, 0, stream>>>(sse, n_seg, n_a, n_r, c1, out);
  return cudaGetLastError();
}

}  // namespace w4

// ---------------------------------------------------------------------------
// Exact tie-breaking of the selections.
//
// The fp16 tensor-core scores are within a small relative error of the
// binary64 definition; a selection whose fp16 values put two or more
// candidates within the tie tolerance of its minimum is decided again on
// binary64 values computed from scratch for exactly those candidates:
//   rowsum[c][n] = sum_m (sum_k (x_mk * fl64(1 / s_k)) (fl64(w_nk s_k) - w_hat_nk))^2
// where w_hat is the candidate's exact dequantized value (the same codes as
// every other path: quant_group.cuh) and w_nk s_k is exact in binary64.
//
// The contraction runs on the fp64 tensor-core MMA (mma.sync m8n8k4; the
// tcgen05 instructions have no binary64 kind): every product and sum is a
// binary64 operation, in a fixed order, so the values do not depend on the
// launch.
// ---------------------------------------------------------------------------
namespace w4 {
namespace {

constexpr int kExactRows = 64;    // weight rows per CTA
constexpr int kExactTok = 128;    // tokens per pass of a CTA
constexpr int kExactChunk = 256;  // tokens per CTA (a grid dimension covers M)
constexpr int kExactLd = 68;      // doubles per smem row: 64 channels + 4 (conflict-free fragments)
constexpr size_t kExactSmem =
    static_cast<size_t>(kExactRows + kExactTok) * kExactLd * sizeof(double) + 128 * sizeof(double);

// D(8x8) += A(8x4) * B(4x8), binary64.  Lane l holds A[l/4][l%4],
// B[l%4][l/4] and D[l/4][2(l%4)], D[l/4][2(l%4)+1].
__device__ __forceinline__ void dmma_m8n8k4(double (&d)[2], double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
               : "+d"(d[0]), "+d"(d[1])
               : "d"(a), "d"(b));
}

// One CTA: 64 weight rows of one listed candidate over one chunk of 256
// tokens (two passes of 128); partial[c][chunk][n] = sum over the chunk's
// tokens of y_mn^2.  Warp w owns rows 32 (w & 1) .. +31 and tokens
// 32 (w >> 1) .. +31 of a pass as 4 x 4 tiles of 8 x 8.  Per group of 128
// channels, threads (r, p) = (t / 4, t % 4) find row r's group statistics
// (channels 32 p .. 32 p + 31, then across the 4 threads); per 64-channel
// half they build row r's error operand for channels 16 p .. 16 p + 15 of
// the half, and thread t scales token t / 2's channels 32 (t % 2) .. +31.
template <bool SYM>
__global__ void __launch_bounds__(256, 2)
    exact_rowsse_kernel(const __nv_bfloat16* __restrict__ x, int M,
                        const __nv_bfloat16* __restrict__ w, int N, int K,
                        const float* __restrict__ s_all, ShrinkList shrinks, int n_r,
                        const int* __restrict__ list, const int* __restrict__ count, int cap,
                        const int* __restrict__ rowlist, const int* __restrict__ rowcount,
                        const uint32_t* __restrict__ cmask, SegOffsets seg, int n_seg,
                        double* __restrict__ partial) {
  extern __shared__ __align__(16) double esm[];
  double* Es = esm;                                // [64 rows][kExactLd]
  double* Xs = esm + kExactRows * kExactLd;        // [128 tokens][kExactLd]
  double* inv_s = Xs + kExactTok * kExactLd;       // [128] 1 / s over the group
  const int ci = blockIdx.z;
  if (ci >= cap || ci >= *count) return;
  const int cand = list[ci];
  const int ia = cand / n_r, jr = cand % n_r;
  const float* s = s_all + static_cast<size_t>(ia) * K;
  const float shrink = shrinks.v[jr];
  const int n0 = blockIdx.x * kExactRows;
  const int t = threadIdx.x;
  // Row i of the tile: n0 + i, or entry n0 + i of the ratio's row list.
  const int nrows = rowlist ? rowcount[jr] : N;
  if (n0 >= nrows) return;
  if (cmask) {  // only the segments whose selections listed this candidate
    const uint32_t m = cmask[ci];
    bool need = false;
    for (int q = 0; q < n_seg; ++q)
      need = need || (((m >> q) & 1u) && seg.off[q] < n0 + kExactRows && seg.off[q + 1] > n0);
    if (!need) return;
  }
  auto row_of = [&](int i) {
    if (n0 + i >= nrows) return -1;
    return rowlist ? rowlist[static_cast<size_t>(jr) * N + n0 + i] : n0 + i;
  };
  const int lane = t & 31, wid = t >> 5;
  const int wn = wid & 1, wm = wid >> 1;
  const int fr = lane >> 2, fq = lane & 3;  // fragment row / k index
  const int r = t >> 2, p = t & 3;
  const int nrow = row_of(r);
  const bool rvalid = nrow >= 0;
  const __nv_bfloat16* wrow = w + static_cast<size_t>(rvalid ? nrow : 0) * K;
  const int G = K / 128;
  const int mbeg = blockIdx.y * kExactChunk;
  const int mend = min(M, mbeg + kExactChunk);
  double rs[4] = {0.0, 0.0, 0.0, 0.0};  // rows 32 wn + 8 i + fr
  for (int m0 = mbeg; m0 < mend; m0 += kExactTok) {
    double acc[4][4][2];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j][0] = acc[i][j][1] = 0.0;
    const int xt = m0 + (t >> 1);  // token this thread scales
    const bool xvalid = xt < mend;
    const __nv_bfloat16* xrow = x + static_cast<size_t>(xvalid ? xt : mbeg) * K;
    for (int g = 0; g < G; ++g) {
      // Group statistics of v = w*s for row r (4 threads x 32 channels).
      float gmax = SYM ? 0.f : -INFINITY, gmin = INFINITY;
      {
        const int kb = 128 * g + 32 * p;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float f8[8];
          bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(wrow + kb) + q), f8);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float v = __fmul_rn(f8[i], __ldg(s + kb + 8 * q + i));
            if (SYM) {
              gmax = fmaxf(gmax, fabsf(v));
            } else {
              gmax = fmaxf(gmax, v);
              gmin = fminf(gmin, v);
            }
          }
        }
      }
#pragma unroll
      for (int o = 1; o <= 2; o <<= 1) {
        gmax = fmaxf(gmax, __shfl_xor_sync(0xffffffffu, gmax, o));
        if (!SYM) gmin = fminf(gmin, __shfl_xor_sync(0xffffffffu, gmin, o));
      }
      const GroupQ gq = group_params<SYM>(gmax, gmin, shrink);
      __syncthreads();  // the previous group's tiles and inv_s are consumed
      if (t < 128) inv_s[t] = 1.0 / static_cast<double>(__ldg(s + 128 * g + t));
      __syncthreads();
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        if (h == 1) __syncthreads();  // half 0's tiles are consumed
        {
          // Row r's error operand, channels 16 p .. 16 p + 15 of the half.
          const int kb = 128 * g + 64 * h + 16 * p;
          double* dst = Es + r * kExactLd + 16 * p;
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            float f8[8];
            bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(wrow + kb) + q), f8);
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
              double d2[2];
#pragma unroll
              for (int u = 0; u < 2; ++u) {
                const float sk = __ldg(s + kb + 8 * q + i + u);
                const float v = __fmul_rn(f8[i + u], sk);
                const float what = __fmul_rn(
                    __fsub_rn(static_cast<float>(code_of(v, gq)), gq.zero), gq.sc);  // exact
                d2[u] = rvalid ? static_cast<double>(f8[i + u]) * static_cast<double>(sk) -
                                     static_cast<double>(what)
                               : 0.0;
              }
              *reinterpret_cast<double2*>(dst + 8 * q + i) = make_double2(d2[0], d2[1]);
            }
          }
        }
        {
          // Token t / 2, channels 32 (t % 2) .. +31 of the half, times 1 / s.
          const int kx = 32 * (t & 1);
          const uint4* xr = reinterpret_cast<const uint4*>(xrow + 128 * g + 64 * h + kx);
          double* dst = Xs + (t >> 1) * kExactLd + kx;
          const double* is = inv_s + 64 * h + kx;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float f8[8];
            bf16x8_to_f32(__ldg(xr + q), f8);
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
              const double a0 = xvalid ? static_cast<double>(f8[i]) * is[8 * q + i] : 0.0;
              const double a1 = xvalid ? static_cast<double>(f8[i + 1]) * is[8 * q + i + 1] : 0.0;
              *reinterpret_cast<double2*>(dst + 8 * q + i) = make_double2(a0, a1);
            }
          }
        }
        __syncthreads();
        const double* ea = Es + (32 * wn + fr) * kExactLd + fq;
        const double* xb = Xs + (32 * wm + fr) * kExactLd + fq;
#pragma unroll 4
        for (int k4 = 0; k4 < 64; k4 += 4) {
          double af[4], bf[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) af[i] = ea[8 * i * kExactLd + k4];
#pragma unroll
          for (int j = 0; j < 4; ++j) bf[j] = xb[8 * j * kExactLd + k4];
#pragma unroll
          for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) dmma_m8n8k4(acc[i][j], af[i], bf[j]);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        rs[i] = fma(acc[i][j][0], acc[i][j][0], rs[i]);
        rs[i] = fma(acc[i][j][1], acc[i][j][1], rs[i]);
      }
  }
  // Row sums: the 4 lanes of a fragment row (fixed butterfly), then the 4
  // token warps in order.
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    rs[i] += __shfl_xor_sync(0xffffffffu, rs[i], 1);
    rs[i] += __shfl_xor_sync(0xffffffffu, rs[i], 2);
  }
  __syncthreads();  // the tiles are consumed; Es holds the warps' sums
  if (fq == 0) {
#pragma unroll
    for (int i = 0; i < 4; ++i) Es[wm * kExactRows + 32 * wn + 8 * i + fr] = rs[i];
  }
  __syncthreads();
  if (t < kExactRows) {
    const int row = row_of(t);
    const double v = ((Es[t] + Es[kExactRows + t]) + Es[2 * kExactRows + t]) + Es[3 * kExactRows + t];
    if (row >= 0) partial[(static_cast<size_t>(ci) * gridDim.y + blockIdx.y) * N + row] = v;
  }
}

// Candidates to decide again for awq_score_grid, as a list of flat ids
// i * n_r + j (at most cap; *count receives the number flagged, which may
// exceed cap).  A selection contributes its near-minimum set only when that
// set has two or more members.  The selections: per segment and for the
// summed table, the joint argmin and alpha* (at the no-clip column c1); per
// segment, shrink* at every alpha that can be a segment's or the group's
// alpha* after the decision.  One block.
__global__ void __launch_bounds__(256)
    awq_flag_kernel(const double* __restrict__ sse, int n_seg, int n_a, int n_r, int c1,
                    double tol, int cap, int* __restrict__ list, int* __restrict__ count,
                    uint32_t* __restrict__ masks) {
  __shared__ uint32_t flag[kMaxGrid * kMaxGrid];  // per candidate: segments that need it
  __shared__ unsigned char near_a[17][kMaxGrid];  // per segment, and the group at n_seg
  __shared__ double dred[8];
  __shared__ int ired[8];
  __shared__ int nflag;
  const int n_c = n_a * n_r;
  const int t = threadIdx.x;
  const int nw = static_cast<int>(blockDim.x >> 5);
  for (int c = t; c < n_c; c += blockDim.x) flag[c] = 0;
  for (int c = t; c < 17 * kMaxGrid; c += blockDim.x) (&near_a[0][0])[c] = 0;
  if (t == 0) nflag = 0;
  __syncthreads();
  // Segment s_ < n_seg, or the summed table (s_ == n_seg).
  auto val = [&](int s_, int c) {
    if (s_ < n_seg) return sse[static_cast<size_t>(s_) * n_c + c];
    double tot = 0.0;
    for (int q = 0; q < n_seg; ++q) tot += sse[static_cast<size_t>(q) * n_c + c];
    return tot;
  };
  auto block_min = [&](double m) {
#pragma unroll
    for (int o = 16; o; o >>= 1) m = fmin(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((t & 31) == 0) dred[t >> 5] = m;
    __syncthreads();
    double r = dred[0];
    for (int i = 1; i < nw; ++i) r = fmin(r, dred[i]);
    __syncthreads();
    return r;
  };
  auto block_sum = [&](int v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if ((t & 31) == 0) ired[t >> 5] = v;
    __syncthreads();
    int r = 0;
    for (int i = 0; i < nw; ++i) r += ired[i];
    __syncthreads();
    return r;
  };
  // One selection: candidates pick(0 .. n-1) of table s_.  Its near-minimum
  // set is marked in `mark` (if given) and flagged when it has >= 2 members,
  // for segment s_ (the summed table: every segment).
  const uint32_t all_seg = n_seg >= 32 ? 0xFFFFFFFFu : (1u << n_seg) - 1u;
  auto decide = [&](auto pick, int n, int s_, unsigned char* mark) {
    const uint32_t bits = s_ < n_seg ? 1u << s_ : all_seg;
    double m = INFINITY;
    for (int u = t; u < n; u += blockDim.x) m = fmin(m, val(s_, pick(u)));
    const double lim = block_min(m) * (1.0 + tol);
    int members = 0;
    for (int u = t; u < n; u += blockDim.x) members += val(s_, pick(u)) <= lim;
    const bool tie = block_sum(members) >= 2;
    for (int u = t; u < n; u += blockDim.x)
      if (val(s_, pick(u)) <= lim) {
        if (mark) mark[u] = 1;
        if (tie) flag[pick(u)] |= bits;
      }
    __syncthreads();
  };
  for (int s_ = 0; s_ <= n_seg; ++s_) {
    decide([](int u) { return u; }, n_c, s_, nullptr);                       // joint
    decide([&](int u) { return u * n_r + c1; }, n_a, s_, near_a[s_]);        // alpha*
  }
  // shrink* per segment at every alpha that may be that segment's or the
  // group's alpha*.
  for (int s_ = 0; s_ < n_seg; ++s_)
    for (int i = 0; i < n_a; ++i)
      if (near_a[s_][i] || near_a[n_seg][i])
        decide([&](int u) { return i * n_r + u; }, n_r, s_, nullptr);
  for (int c = t; c < n_c; c += blockDim.x)
    if (flag[c]) {
      const int slot = atomicAdd(&nflag, 1);
      if (slot < cap) {
        list[slot] = c;
        masks[slot] = flag[c];
      }
    }
  __syncthreads();
  if (t == 0) *count = nflag;
}

// Writes the exact values of the decided candidates into the table:
// sse[seg][c] = sum over the segment's rows, in order, of rowsum.
__global__ void awq_exact_merge_kernel(const double* __restrict__ partial, int chunks, int N,
                                       const int* __restrict__ list, const int* __restrict__ count,
                                       const uint32_t* __restrict__ masks, int cap, int n_seg,
                                       SegOffsets seg, int n_c, double* __restrict__ sse) {
  const int ci = blockIdx.x;
  const int n = *count < cap ? *count : cap;
  if (ci >= n) return;
  const int s_ = threadIdx.x;
  if (s_ >= n_seg || !((masks[ci] >> s_) & 1u)) return;  // a segment not recomputed
  double sum = 0.0;
  for (int row = seg.off[s_]; row < seg.off[s_ + 1]; ++row) {
    double rsum = 0.0;
    for (int c = 0; c < chunks; ++c)
      rsum += partial[(static_cast<size_t>(ci) * chunks + c) * N + row];
    sum += rsum;
  }
  sse[static_cast<size_t>(s_) * n_c + list[ci]] = sum;
}

// Per-output-channel clipping: near ties per row.  flags[j][n] = 1 when row
// n has two or more ratios within tol of its least fp16 value and j is one of
// them; mask bit j is set if any row flags j.  One thread per row.
__global__ void clip_flag_kernel(const double* __restrict__ sse_rows, int64_t N, int n_r,
                                 double tol, uint8_t* __restrict__ flags,
                                 unsigned long long* __restrict__ mask) {
  const int64_t n = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (n >= N) return;
  double mn = INFINITY;
  for (int j = 0; j < n_r; ++j) mn = fmin(mn, sse_rows[static_cast<size_t>(j) * N + n]);
  int members = 0;
  for (int j = 0; j < n_r; ++j) members += sse_rows[static_cast<size_t>(j) * N + n] <= mn * (1.0 + tol);
  unsigned long long bits = 0;
  for (int j = 0; j < n_r; ++j) {
    const bool f = members >= 2 && sse_rows[static_cast<size_t>(j) * N + n] <= mn * (1.0 + tol);
    flags[static_cast<size_t>(j) * N + n] = f;
    if (f) bits |= 1ull << j;
  }
  if (bits) atomicOr(mask, bits);
}

// The ratios any row needs decided again, as candidate ids (alpha index 0).
__global__ void clip_list_kernel(const unsigned long long* __restrict__ mask, int n_r,
                                 int* __restrict__ list, int* __restrict__ count) {
  if (threadIdx.x != 0) return;
  int c = 0;
  for (int j = 0; j < n_r; ++j)
    if ((*mask >> j) & 1ull) list[c++] = j;
  *count = c;
}

// rows[j][0 .. counts[j]) = the rows that flag ratio j, ascending.  One
// block per ratio (1024 threads), a block-wide scan per 1024 rows.
__global__ void __launch_bounds__(1024)
    clip_compact_kernel(const uint8_t* __restrict__ flags, int64_t N, int* __restrict__ rows,
                        int* __restrict__ counts) {
  __shared__ int wsum[32];
  __shared__ int base;
  const int j = blockIdx.x;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int nw = static_cast<int>(blockDim.x >> 5);
  const uint8_t* f = flags + static_cast<size_t>(j) * N;
  int* out = rows + static_cast<size_t>(j) * N;
  if (t == 0) base = 0;
  __syncthreads();
  for (int64_t c0 = 0; c0 < N; c0 += blockDim.x) {
    const int64_t n = c0 + t;
    const int v = (n < N && f[n]) ? 1 : 0;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int ws = lane < nw ? wsum[lane] : 0;
      int wi = ws;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, wi, o);
        if (lane >= o) wi += y;
      }
      if (lane < nw) wsum[lane] = wi - ws;  // exclusive
    }
    __syncthreads();
    const int pos = base + wsum[warp] + incl - v;
    if (v) out[pos] = static_cast<int>(n);
    __syncthreads();  // every thread has read base
    if (t == static_cast<int>(blockDim.x) - 1) base = pos + v;
    __syncthreads();
  }
  if (t == 0) counts[j] = base;
}

// Flagged rows take the exact values of their flagged ratios and choose
// again (lowest index on equal values).  One thread per row.
__global__ void clip_exact_merge_kernel(const double* __restrict__ partial, int chunks,
                                        const uint8_t* __restrict__ flags,
                                        const int* __restrict__ list, const int* __restrict__ count,
                                        int64_t N, int n_r, ShrinkList shrinks,
                                        double* __restrict__ sse_rows,
                                        int32_t* __restrict__ choice,
                                        float* __restrict__ shrink_rows) {
  const int64_t n = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (n >= N) return;
  bool any = false;
  for (int ci = 0; ci < *count; ++ci) {
    const int j = list[ci];
    if (flags[static_cast<size_t>(j) * N + n]) {
      double v = 0.0;
      for (int c = 0; c < chunks; ++c) v += partial[(static_cast<size_t>(ci) * chunks + c) * N + n];
      sse_rows[static_cast<size_t>(j) * N + n] = v;
      any = true;
    }
  }
  if (!any) return;
  int best = 0;
  double best_v = sse_rows[n];
  for (int j = 1; j < n_r; ++j) {
    const double v = sse_rows[static_cast<size_t>(j) * N + n];
    if (v < best_v) {
      best = j;
      best_v = v;
    }
  }
  choice[n] = best;
  if (shrink_rows) shrink_rows[n] = shrinks.v[best];
}

template <auto kern>
cudaError_t exact_smem_attr() {
  static unsigned long long done = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 64 && (__atomic_load_n(&done, __ATOMIC_ACQUIRE) & (1ull << dev))) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kExactSmem));
  if (e == cudaSuccess && dev < 64) __atomic_fetch_or(&done, 1ull << dev, __ATOMIC_RELEASE);
  return e;
}

}  // namespace

int exact_token_chunks(int M) { return (M + kExactChunk - 1) / kExactChunk; }

cudaError_t launch_exact_rowsse(const void* x, int M, const void* w, int N, int K,
                                const float* s_all, const ShrinkList& shrinks, int n_r,
                                bool symmetric, const int* list, const int* count, int cap,
                                const int* rowlist, const int* rowcount, const uint32_t* cmask,
                                const SegOffsets& seg, int n_seg, double* rowsum,
                                cudaStream_t stream) {
  const dim3 grid(static_cast<unsigned>((N + kExactRows - 1) / kExactRows),
                  static_cast<unsigned>(exact_token_chunks(M)), static_cast<unsigned>(cap));
  const auto* xb = static_cast<const __nv_bfloat16*>(x);
  const auto* wb = static_cast<const __nv_bfloat16*>(w);
  cudaError_t e;
  if (symmetric) {
    e = exact_smem_attr<exact_rowsse_kernel<true>>();
    if (e != cudaSuccess) return e;
    exact_rowsse_kernel<true><<<grid, 256, kExactSmem, stream>>>(
        xb, M, wb, N, K, s_all, shrinks, n_r, list, count, cap, rowlist, rowcount, cmask, seg,
        n_seg, rowsum);
  } else {
    e = exact_smem_attr<exact_rowsse_kernel<false>>();
    if (e != cudaSuccess) return e;
    exact_rowsse_kernel<false><<<grid, 256, kExactSmem, stream>>>(
        xb, M, wb, N, K, s_all, shrinks, n_r, list, count, cap, rowlist, rowcount, cmask, seg,
        n_seg, rowsum);
  }
  return cudaGetLastError();
}

cudaError_t launch_awq_flag(const double* sse, int n_seg, int n_a, int n_r, int c1, double tol,
                            int cap, int* list, int* count, uint32_t* masks, cudaStream_t stream) {
  awq_flag_kernel<<<1, 256, 0, stream>>>(sse, n_seg, n_a, n_r, c1, tol, cap, list, count, masks);
  return cudaGetLastError();
}

cudaError_t launch_awq_exact_merge(const double* rowsum, int M, int N, const int* list,
                                   const int* count, const uint32_t* masks, int cap, int n_seg,
                                   const SegOffsets& seg, int n_c, double* sse,
                                   cudaStream_t stream) {
  awq_exact_merge_kernel<<<cap, 32, 0, stream>>>(rowsum, exact_token_chunks(M), N, list, count,
                                                 masks, cap, n_seg, seg, n_c, sse);
  return cudaGetLastError();
}

cudaError_t launch_clip_exact(const void* x, int M, const void* w, int N, int K, const float* s,
                              const ShrinkList& shrinks, bool symmetric, double tol,
                              double* sse_rows, int32_t* choice, float* shrink_rows,
                              uint8_t* flags, unsigned long long* mask, int* list, int* count,
                              int* rows, int* row_counts, double* rowsum, cudaStream_t stream) {
  cudaError_t e = cudaMemsetAsync(mask, 0, sizeof(unsigned long long), stream);
  if (e != cudaSuccess) return e;
  const unsigned blocks = static_cast<unsigned>((N + 127) / 128);
  clip_flag_kernel<<<blocks, 128, 0, stream>>>(sse_rows, N, shrinks.n, tol, flags, mask);
  clip_list_kernel<<<1, 32, 0, stream>>>(mask, shrinks.n, list, count);
  clip_compact_kernel<<<shrinks.n, 1024, 0, stream>>>(flags, N, rows, row_counts);
  e = launch_exact_rowsse(x, M, w, N, K, s, shrinks, shrinks.n, symmetric, list, count, shrinks.n,
                          rows, row_counts, nullptr, SegOffsets{}, 0, rowsum, stream);
  if (e != cudaSuccess) return e;
  clip_exact_merge_kernel<<<blocks, 128, 0, stream>>>(rowsum, exact_token_chunks(M), flags, list,
                                                      count, N, shrinks.n, shrinks, sse_rows,
                                                      choice, shrink_rows);
  return cudaGetLastError();
}

}  // namespace w4
