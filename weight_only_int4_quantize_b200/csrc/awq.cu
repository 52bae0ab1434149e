// AWQ alpha x shrink candidate scoring ("ghostchoir/rebuttal_w4g128_awq_w2"
// model card, 'Model Details' row 'Search' and the scale-rewrite paragraph).
//
// For each alpha_i the scales s = max(mean_m |x_m|, 1e-8)^alpha_i are formed
// once; the candidate error of shrink r_j is scored in the s-domain,
//   x . (W - dequant(Q_r(W diag(s))) diag(1/s))^T
//     = (x diag(1/s)) . (W diag(s) - dequant(Q_r(W diag(s))))^T,
// which keeps both tensor-core operands well scaled for fp16:
//   A_i = fp16(x / s)              [M, K]   (awq_xs_kernel)
//   E_ij = fp16(w*s - w_hat)       [N, K]   (awq_err_kernel, all shrinks of
//                                             one alpha in one pass over W)
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

// A = fp16(x / s), correctly rounded binary32 division, then fp16 RNE.
__global__ void awq_xs_kernel(const __nv_bfloat16* __restrict__ x, const float* __restrict__ s,
                              int64_t M, int64_t K, __half* __restrict__ a) {
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
      const __half2 h = __halves2half2(__float2half_rn(__fdiv_rn(v[2 * p], sv[2 * p])),
                                       __float2half_rn(__fdiv_rn(v[2 * p + 1], sv[2 * p + 1])));
      o[p] = *reinterpret_cast<const uint32_t*>(&h);
    }
    reinterpret_cast<uint4*>(a)[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// E_j[n, k] = fp16(v - w_hat) with v = w*s and w_hat = (q - zero)*scale the
// candidate's exact dequantized value, for every shrink j, one half warp per
// 128-value group (same lane layout as the quantize kernel).
template <bool SYM>
__global__ void __launch_bounds__(256)
    awq_err_kernel(const uint4* __restrict__ w, const float* __restrict__ s, int64_t n_groups,
                   int64_t groups_per_row, ShrinkList shrinks, int64_t plane_elems,
                   __half* __restrict__ e) {
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
          d[h] = __fsub_rn(val, what);
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

// SSE[seg, i, j] = sum over tiles (fixed order) of the GEMM's tile sums.
__global__ void awq_reduce_kernel(const double* __restrict__ partials, int n_cand, int n_seg,
                                  int tiles, double* __restrict__ sse) {
  const int id = blockIdx.x * blockDim.x + threadIdx.x;  // = seg * n_cand + cand
  if (id >= n_cand * n_seg) return;
  const int seg = id / n_cand;
  const int cand = id % n_cand;
  const double* p = partials + (static_cast<size_t>(cand) * n_seg + seg) * tiles;
  double sum = 0.0;
  for (int t = 0; t < tiles; ++t) sum += p[t];
  sse[id] = sum;
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
                                        double* __restrict__ sse_rows, int32_t* __restrict__ choice,
                                        float* __restrict__ shrink_rows) {
  const int64_t n = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (n >= N) return;
  int best = 0;
  double best_v = 0.0;
  for (int c = 0; c < n_cand; ++c) {
    double v = 0.0;
    for (int t = 0; t < row_tiles; ++t) v += partials[(static_cast<size_t>(c) * row_tiles + t) * N + n];
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
                                    const ShrinkList& shrinks, double* sse_rows, int32_t* choice,
                                    float* shrink_rows, cudaStream_t stream) {
  const int64_t blocks = (N + 127) / 128;
  clip_rows_select_kernel<<<static_cast<unsigned>(blocks), 128, 0, stream>>>(
      partials, n_cand, row_tiles, N, shrinks, sse_rows, choice, shrink_rows);
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

cudaError_t launch_awq_xs(const void* x, const float* s, int64_t M, int64_t K, void* a,
                          cudaStream_t stream, int num_sms) {
  const int64_t n8 = M * K / 8;
  int64_t blocks = (n8 + 255) / 256;
  if (blocks > static_cast<int64_t>(num_sms) * 8) blocks = static_cast<int64_t>(num_sms) * 8;
  awq_xs_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(x), s, M, K, static_cast<__half*>(a));
  return cudaGetLastError();
}

cudaError_t launch_awq_err(const void* w, const float* s, int64_t N, int64_t K, bool symmetric,
                           const ShrinkList& shrinks, void* e, cudaStream_t stream, int num_sms) {
  const int64_t n_groups = N * (K / 128);
  const int64_t n_units = (n_groups + 1) / 2;
  int64_t blocks = (n_units + 7) / 8;
  if (blocks > static_cast<int64_t>(num_sms) * 8) blocks = static_cast<int64_t>(num_sms) * 8;
  const uint4* wp = static_cast<const uint4*>(w);
  __half* ep = static_cast<__half*>(e);
  if (symmetric)
    awq_err_kernel<true><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        wp, s, n_groups, K / 128, shrinks, N * K, ep);
  else
    awq_err_kernel<false><<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
        wp, s, n_groups, K / 128, shrinks, N * K, ep);
  return cudaGetLastError();
}

cudaError_t launch_awq_reduce(const double* partials, int n_cand, int n_seg, int tiles,
                              double* sse, cudaStream_t stream) {
  const int n = n_cand * n_seg;
  awq_reduce_kernel<<<(n + 127) / 128, 128, 0, stream>>>(partials, n_cand, n_seg, tiles, sse);
  return cudaGetLastError();
}

cudaError_t launch_awq_argmin(const double* sse, int n_seg, int n_a, int n_r, int c1,
                              int32_t* out, cudaStream_t stream) {
  awq_argmin_kernel<<<1, 32, 0, stream>>>(sse, n_seg, n_a, n_r, c1, out);
  return cudaGetLastError();
}

}  // namespace w4
