// Block-level AWQ candidate scoring in binary64: one Qwen3-style decoder
// block (and optionally its successor) run forward with a candidate's
// quantized linears swapped in, the loss taken against the unquantized
// path.
//
// Definition ("ghostchoir/rebuttal_w4g128_awq_w2" model card): the 'Search'
// row of the 'Model Details' table (AWQ scale exponent on a 20-point grid,
// a 10-point shrink grid); the paragraph under that table (a candidate for
// block i is scored at the output of block i+1, which stays in original
// precision, against the same path with block i unquantized; the last block
// falls back to its own output); the scale-rewrite paragraph (a candidate
// swaps only the linear's weight, Q(W diag(s)) diag(1/s)); 'Clipping
// granularity' (one shrink ratio per linear); the perplexity table's d=0
// row (the loss at block i's own output).  Block shapes: the
// "ariacompute/qwen3-1.7b_q326_channel" page (16 query heads, 8 key/value
// heads of width 128, SwiGLU width 6144).
//
// The decoder block itself is not on the pages; it follows the published
// Qwen3 conventions: pre-norm, RMSNorm (eps 1e-6) also per head on q and k
// before a rotate-half rotary embedding (theta 1e6), causal softmax
// attention scaled by 1/sqrt(d) with grouped key/value heads, a SwiGLU MLP,
// residual adds.  The AWQ statistic of a linear group is the mean |input|
// over tokens of the activation entering the group on the unquantized
// path; s = fp32(max(stat, 1e-8)^alpha).
//
// Everything runs in binary64: the contractions on the fp64 tensor-core MMA
// (mma.sync m8n8k4, in a fixed order per output), the rest in IEEE double
// with the operations in the definition's order (no contraction where the
// definition rounds twice), so the losses are those of the definition up to
// the order of the sums.
#include <algorithm>
#include <cmath>
#include <cstdint>

#include "quant_group.cuh"
#include "w4_common.cuh"
#include "w4_kernels.h"

namespace w4 {
namespace {

// ---------------------------------------------------------------------------
// Batched fp64 GEMM: C[b] (+)= A[b] B[b / bdiv]^T (+ R) with arbitrary
// strides.  CTA tile 64 (M) x 128 (N); 32-deep k steps staged in shared
// memory by asynchronous copies, two stages (the next step's copies are in
// flight while this one's MMAs run); warp w owns rows 32 (w & 1) .. +31 and
// columns 32 (w >> 1) .. +31 as 4 x 4 MMA tiles of 8 x 8.  A and a binary64
// B are staged as doubles; a bf16 B (k contiguous) is staged as raw bf16 and
// widened when its fragments are loaded (exact).
// ---------------------------------------------------------------------------
constexpr int kGM = 64, kGN = 128, kGK = 32;
constexpr int kGLd = 36;   // doubles per staged row (32 + 4: conflict-free fragment loads)
constexpr int kGLdH = 40;  // bf16 per staged row (32 + 8: conflict-free fragment loads)
constexpr uint32_t kStageA = kGM * kGLd * 8;
constexpr uint32_t kStageBd = kGN * kGLd * 8;
constexpr uint32_t kStageBh = kGN * kGLdH * 2;
template <typename TB>
__host__ __device__ constexpr uint32_t gemm_stage_bytes() {
  return kStageA + (sizeof(TB) == 8 ? kStageBd : kStageBh);
}
template <typename TB>
constexpr size_t gemm_smem_bytes() {
  return 2 * static_cast<size_t>(gemm_stage_bytes<TB>());
}

struct GemmArgs {
  const double* A;
  int64_t sAm, sAk, bA;
  const void* B;  // double, or bf16 bits with sBk == 1
  int64_t sBn, sBk, bB;
  int bdiv;  // batch b reads B batch b / bdiv
  double* C;
  int64_t sCm, sCn, bC;
  const double* R;  // optional residual, same strides as C
  int M, N, K;
  int causal;  // 1: skip tiles with every column above every row; 2: k < row tile end
};

__device__ __forceinline__ void dmma_m8n8k4(double (&d)[2], double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
               : "+d"(d[0]), "+d"(d[1])
               : "d"(a), "d"(b));
}

// Asynchronous copies global -> shared of 8 / 4 bytes; nothing is read (the
// destination is zero-filled) when `valid` is false.
__device__ __forceinline__ void cpa8(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 8 : 0)
               : "memory");
}
__device__ __forceinline__ void cpa4(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 4 : 0)
               : "memory");
}
__device__ __forceinline__ void cpa_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cpa_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Stages rows [r0, r0 + ROWS) x channels [k0, k0 + 32) of a strided binary64
// operand (zero outside [0, nrows) x [0, kend)) as dst[row][kGLd].
template <int ROWS>
__device__ __forceinline__ void stage_f64(uint32_t dst, const double* src, int64_t s_row,
                                          int64_t s_k, int r0, int nrows, int k0, int kend) {
  const int t = threadIdx.x;
  constexpr int kPer = ROWS * kGK / 256;
  if (s_k == 1) {  // lanes along k: a warp copies 256 contiguous bytes
    const int kk = t & 31;
    const int k = k0 + kk;
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int r = (t >> 5) + 8 * j;
      const int row = r0 + r;
      const bool v = row < nrows && k < kend;
      cpa8(dst + static_cast<uint32_t>(r * kGLd + kk) * 8u, v ? src + row * s_row + k : src, v);
    }
  } else {  // lanes along rows
    constexpr int kStep = 256 / ROWS;
    const int r = t % ROWS;
    const int row = r0 + r;
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
      const int kk = t / ROWS + kStep * j;
      const int k = k0 + kk;
      const bool v = row < nrows && k < kend;
      cpa8(dst + static_cast<uint32_t>(r * kGLd + kk) * 8u,
           v ? src + row * s_row + k * s_k : src, v);
    }
  }
}

// Stages 128 rows x 32 channels of a bf16 operand with k contiguous (K and
// k0 even) as raw bf16 pairs, dst[row][kGLdH].
__device__ __forceinline__ void stage_bf16(uint32_t dst, const uint16_t* src, int64_t s_row,
                                           int r0, int nrows, int k0, int kend) {
  const int t = threadIdx.x;
  const int pr = t & 15;
  const int k = k0 + 2 * pr;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int r = (t >> 4) + 16 * j;
    const int row = r0 + r;
    const bool v = row < nrows && k < kend;
    cpa4(dst + static_cast<uint32_t>(r * kGLdH + 2 * pr) * 2u, v ? src + row * s_row + k : src, v);
  }
}

__device__ __forceinline__ double bf16_bits_to_double(uint16_t h) {
  return static_cast<double>(__uint_as_float(static_cast<uint32_t>(h) << 16));
}

template <typename TB>
__global__ void __launch_bounds__(256, 2) gemm_f64_kernel(GemmArgs g) {
  constexpr bool kBf16 = sizeof(TB) == 2;
  extern __shared__ __align__(16) uint8_t gsm[];
  const uint32_t sbase = smem_u32(gsm);
  const int m0 = blockIdx.y * kGM, n0 = blockIdx.x * kGN;
  if (g.causal == 1 && n0 >= m0 + kGM) return;  // every key after every query
  const int b = blockIdx.z;
  const double* A = g.A + b * g.bA;
  const TB* B = static_cast<const TB*>(g.B) + (b / g.bdiv) * g.bB;
  const int kend = g.causal == 2 ? min(g.K, m0 + kGM) : g.K;
  const int nk = (kend + kGK - 1) / kGK;
  const int t = threadIdx.x, lane = t & 31, wid = t >> 5;
  const int wr = wid & 1, wc = wid >> 1;
  const int fr = lane >> 2, fq = lane & 3;
  auto stage = [&](int buf, int k0) {
    const uint32_t st = sbase + buf * gemm_stage_bytes<TB>();
    stage_f64<kGM>(st, A, g.sAm, g.sAk, m0, g.M, k0, kend);
    if constexpr (kBf16)
      stage_bf16(st + kStageA, reinterpret_cast<const uint16_t*>(B), g.sBn, n0, g.N, k0, kend);
    else
      stage_f64<kGN>(st + kStageA, reinterpret_cast<const double*>(B), g.sBn, g.sBk, n0, g.N, k0,
                     kend);
  };
  double acc[4][4][2];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j][0] = acc[i][j][1] = 0.0;
  if (nk > 0) stage(0, 0);
  cpa_commit();
  for (int kt = 0; kt < nk; ++kt) {
    if (kt + 1 < nk) {
      stage((kt + 1) & 1, (kt + 1) * kGK);  // its buffer was consumed at step kt - 1
      cpa_commit();
      cpa_wait<1>();
    } else {
      cpa_wait<0>();
    }
    __syncthreads();  // every thread's copies of step kt have landed
    const uint8_t* st = gsm + (kt & 1) * gemm_stage_bytes<TB>();
    const double* ea = reinterpret_cast<const double*>(st) + (32 * wr + fr) * kGLd + fq;
#pragma unroll
    for (int k4 = 0; k4 < kGK; k4 += 4) {
      double af[4], bf[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) af[i] = ea[8 * i * kGLd + k4];
      if constexpr (kBf16) {
        const uint16_t* eb =
            reinterpret_cast<const uint16_t*>(st + kStageA) + (32 * wc + fr) * kGLdH + fq;
#pragma unroll
        for (int j = 0; j < 4; ++j) bf[j] = bf16_bits_to_double(eb[8 * j * kGLdH + k4]);
      } else {
        const double* eb =
            reinterpret_cast<const double*>(st + kStageA) + (32 * wc + fr) * kGLd + fq;
#pragma unroll
        for (int j = 0; j < 4; ++j) bf[j] = eb[8 * j * kGLd + k4];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) dmma_m8n8k4(acc[i][j], af[i], bf[j]);
    }
    __syncthreads();  // step kt's buffer is consumed before step kt + 2 refills it
  }
  double* C = g.C + b * g.bC;
  const double* R = g.R ? g.R + b * g.bC : nullptr;  // never the output itself
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + 32 * wr + 8 * i + fr;
    if (m >= g.M) continue;
    // The row's eight residual values are loaded before its stores.
    double rv[4][2];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int n = n0 + 32 * wc + 8 * j + 2 * fq + u;
        rv[j][u] = (R && n < g.N) ? __ldg(R + m * g.sCm + n * g.sCn) : 0.0;
      }
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int n = n0 + 32 * wc + 8 * j + 2 * fq + u;
        if (n >= g.N) continue;
        const int64_t o = m * g.sCm + n * g.sCn;
        C[o] = R ? __dadd_rn(rv[j][u], acc[i][j][u]) : acc[i][j][u];
      }
  }
}

// ---------------------------------------------------------------------------
// Elementwise and row kernels
// ---------------------------------------------------------------------------
// Sum over the block (256 threads) in a fixed order.
__device__ __forceinline__ double block_sum256(double v, double* red) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  double s = 0.0;
#pragma unroll
  for (int i = 0; i < 8; ++i) s += red[i];
  __syncthreads();
  return s;
}

// out = x / sqrt(mean(x^2) + eps) * gamma per row of D; one block per row.
__global__ void __launch_bounds__(256)
    rmsnorm_f64_kernel(const double* __restrict__ x, const double* __restrict__ gamma, int D,
                       double eps, double* __restrict__ out) {
  __shared__ double red[8];
  const double* xr = x + static_cast<int64_t>(blockIdx.x) * D;
  double* yr = out + static_cast<int64_t>(blockIdx.x) * D;
  double ss = 0.0;
  for (int k = threadIdx.x; k < D; k += 256) ss = fma(xr[k], xr[k], ss);
  ss = block_sum256(ss, red);
  const double r = sqrt(__dadd_rn(ss / D, eps));
  for (int k = threadIdx.x; k < D; k += 256) yr[k] = __dmul_rn(xr[k] / r, gamma[k]);
}

// Per head: RMSNorm over the head's d channels, then the rotary embedding
// at the token's position (rotate half: channels i and i + d/2, i < d/2,
// turn by p * theta^(-2i/d)).  One warp per (token, head), in place; E =
// d / 32 channels per lane (lane + 32 j).
template <int E>
__global__ void __launch_bounds__(256)
    qknorm_rope_kernel(const double* xin, double* x, int64_t rows, int heads,
                       const double* __restrict__ gain, double eps, double theta) {
  constexpr int d = 32 * E;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int lane = threadIdx.x & 31;
  const int64_t pos = row / heads;
  const double* xi = xin + row * d;  // may be x itself
  double* xr = x + row * d;
  double v[E];
  double ss = 0.0;
#pragma unroll
  for (int j = 0; j < E; ++j) {
    v[j] = xi[lane + 32 * j];
    ss = fma(v[j], v[j], ss);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const double r = sqrt(__dadd_rn(ss / d, eps));
#pragma unroll
  for (int j = 0; j < E; ++j) v[j] = __dmul_rn(v[j] / r, gain[lane + 32 * j]);
#pragma unroll
  for (int j = 0; j < E / 2; ++j) {
    const int i = lane + 32 * j;
    const double inv = pow(theta, (-2.0 * i) / d);
    const double ang = __dmul_rn(static_cast<double>(pos), inv);
    double sn, cs;
    sincos(ang, &sn, &cs);
    const double x1 = v[j], x2 = v[j + E / 2];
    xr[i] = __dsub_rn(__dmul_rn(x1, cs), __dmul_rn(x2, sn));
    xr[i + d / 2] = __dadd_rn(__dmul_rn(x2, cs), __dmul_rn(x1, sn));
  }
}

// Causal softmax of one score row in place: s_j = S_j / sqrt(d) for
// j <= t, p_j = exp(s_j - max) / sum; p_j = 0 for j > t.  One warp per
// (head, query t).
__global__ void __launch_bounds__(256)
    softmax_causal_kernel(double* __restrict__ S, int64_t rows, int T, double sqrt_d) {
  const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int lane = threadIdx.x & 31;
  const int t = static_cast<int>(row % T);
  double* sr = S + row * T;
  double mx = -INFINITY;
  for (int j = lane; j <= t; j += 32) mx = fmax(mx, sr[j] / sqrt_d);
#pragma unroll
  for (int o = 16; o; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  double sum = 0.0;
  for (int j = lane; j <= t; j += 32) sum += exp(__dsub_rn(sr[j] / sqrt_d, mx));
#pragma unroll
  for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  for (int j = lane; j < T; j += 32)
    sr[j] = j <= t ? exp(__dsub_rn(sr[j] / sqrt_d, mx)) / sum : 0.0;
}

// act = silu(g) * u, silu(z) = z / (1 + exp(-z)).
__global__ void swiglu_f64_kernel(const double* __restrict__ g, const double* __restrict__ u,
                                  double* __restrict__ act, int64_t n) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const double z = g[i];
    act[i] = __dmul_rn(z / __dadd_rn(1.0, exp(-z)), u[i]);
  }
}

// stat[k] = mean over the T rows of |a[t][k]|.
__global__ void colmean_abs_f64_kernel(const double* __restrict__ a, int T, int K,
                                       double* __restrict__ stat) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= K) return;
  double s = 0.0;
  for (int t = 0; t < T; ++t) s += fabs(a[static_cast<int64_t>(t) * K + k]);
  stat[k] = s / T;
}

// s[k] = fp32(max(stat[k], 1e-8) ^ alpha), alpha = alphas[ia] with ia the
// constant `index` or, if idx is given, idx[0].
__global__ void block_scales_kernel(const double* __restrict__ stat, int K, AlphaList alphas,
                                    int index, const int32_t* __restrict__ idx,
                                    float* __restrict__ s) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= K) return;
  const float a = alphas.v[idx ? idx[0] : index];
  s[k] = static_cast<float>(pow(fmax(stat[k], 1e-8), static_cast<double>(a)));
}

// The candidate weight Q_r(W diag(s)) diag(1/s) in binary64: one warp per
// (row, group of 128), lane l holds channels 4l .. 4l + 3 of the group.
// Codes and scales are those of quant_group.cuh (the deployed quantizer).
// DELTA: out = that weight minus W (binary64), the change a candidate makes.
template <bool SYM, bool DELTA = false>
__global__ void __launch_bounds__(256)
    candidate_weight_kernel(const uint16_t* __restrict__ w, int N, int K,
                            const float* __restrict__ s, float shrink,
                            double* __restrict__ out) {
  const int G = K / 128;
  const int64_t item = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (item >= static_cast<int64_t>(N) * G) return;
  const int lane = threadIdx.x & 31;
  const int64_t n = item / G;
  const int k0 = static_cast<int>(item % G) * 128 + 4 * lane;
  float wf[4], sk[4], v[4];
  float gmax = SYM ? 0.f : -INFINITY, gmin = INFINITY;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    wf[i] = __uint_as_float(static_cast<uint32_t>(w[n * K + k0 + i]) << 16);
    sk[i] = s[k0 + i];
    v[i] = __fmul_rn(wf[i], sk[i]);
    if (SYM) {
      gmax = fmaxf(gmax, fabsf(v[i]));
    } else {
      gmax = fmaxf(gmax, v[i]);
      gmin = fminf(gmin, v[i]);
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    gmax = fmaxf(gmax, __shfl_xor_sync(0xffffffffu, gmax, o));
    if (!SYM) gmin = fminf(gmin, __shfl_xor_sync(0xffffffffu, gmin, o));
  }
  const GroupQ gq = group_params<SYM>(gmax, gmin, shrink);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float what =
        __fmul_rn(__fsub_rn(static_cast<float>(code_of(v[i], gq)), gq.zero), gq.sc);  // exact
    const double wc = static_cast<double>(what) / static_cast<double>(sk[i]);
    out[n * K + k0 + i] = DELTA ? __dsub_rn(wc, static_cast<double>(wf[i])) : wc;
  }
}

constexpr int kLossBlocks = 296;

// A selection of the search decides in binary64 among the candidates whose
// screening loss is within this relative distance of the least.  The
// screening losses differ from the binary64 ones by far less (the fp16
// roundings touch only each linear's change, about 2^-11 of it, and the
// loss averages them over every token and hidden unit): at most 4.3e-5 on
// Qwen3-1.7B-shaped blocks at 256 and 2048 tokens, both arms.  Outlier
// input channels concentrate the rounding on a few terms (on the fp16 AWQ
// grid they raised the error about 5x), so half of the tolerance keeps a
// margin above that too; the tests hold the difference below half of it,
// with and without outlier channels.
constexpr double kBlockTieTol = 1e-3;

// Per-block partial sums of (a - b)^2 (grid of kLossBlocks blocks).
__global__ void __launch_bounds__(256)
    sqdiff_partial_kernel(const double* __restrict__ a, const double* __restrict__ b, int64_t n,
                          double* __restrict__ partial) {
  __shared__ double red[8];
  double s = 0.0;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; i < n;
       i += static_cast<int64_t>(kLossBlocks) * 256) {
    const double d = __dsub_rn(a[i], b[i]);
    s = fma(d, d, s);
  }
  s = block_sum256(s, red);
  if (threadIdx.x == 0) partial[blockIdx.x] = s;
}

// out[0] = (sum of the partials in order) / n.
__global__ void loss_finish_kernel(const double* __restrict__ partial, int64_t n,
                                   double* __restrict__ out) {
  if (threadIdx.x != 0) return;
  double s = 0.0;
  for (int i = 0; i < kLossBlocks; ++i) s += partial[i];
  out[0] = s / static_cast<double>(n);
}

// ---------------------------------------------------------------------------
// Screening kernels: fp16 tensor-core operands with power-of-two scaling
// ---------------------------------------------------------------------------
// partial[b] = max |a - b| (b may be null) over block b's grid-stride part.
__global__ void __launch_bounds__(256)
    absmax_partial_kernel(const double* __restrict__ a, const double* __restrict__ b, int64_t n,
                          double* __restrict__ partial) {
  __shared__ double red[8];
  double m = 0.0;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; i < n;
       i += static_cast<int64_t>(kLossBlocks) * 256)
    m = fmax(m, fabs(b ? __dsub_rn(a[i], b[i]) : a[i]));
#pragma unroll
  for (int o = 16; o; o >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    double r = red[0];
    for (int i = 1; i < 8; ++i) r = fmax(r, red[i]);
    partial[blockIdx.x] = r;
  }
}

__global__ void __launch_bounds__(256)
    absmax_partial_bf16_kernel(const uint16_t* __restrict__ w, int64_t n,
                               double* __restrict__ partial) {
  __shared__ double red[8];
  float m = 0.f;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; i < n;
       i += static_cast<int64_t>(kLossBlocks) * 256)
    m = fmaxf(m, fabsf(__uint_as_float(static_cast<uint32_t>(w[i]) << 16)));
#pragma unroll
  for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    double r = red[0];
    for (int i = 1; i < 8; ++i) r = fmax(r, red[i]);
    partial[blockIdx.x] = r;
  }
}

// The exponent e that puts the largest magnitude in [2^14, 2^15) (0 for an
// all-zero tensor), from the partial maxima.
__device__ __forceinline__ int f16_exponent(const double* __restrict__ partial) {
  double m = 0.0;
  for (int i = 0; i < kLossBlocks; ++i) m = fmax(m, partial[i]);
  return m > 0.0 ? 14 - ilogb(m) : 0;
}

// out = fp16((a - b) * 2^e) (b may be null); *e_out = e.
__global__ void __launch_bounds__(256)
    to_f16_kernel(const double* __restrict__ a, const double* __restrict__ b, int64_t n,
                  const double* __restrict__ partial, int* __restrict__ e_out,
                  __half* __restrict__ out) {
  __shared__ int se;
  if (threadIdx.x == 0) {
    se = f16_exponent(partial);
    if (blockIdx.x == 0) *e_out = se;
  }
  __syncthreads();
  const int e = se;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * 256)
    out[i] = __double2half(ldexp(b ? __dsub_rn(a[i], b[i]) : a[i], e));
}

__global__ void __launch_bounds__(256)
    bf16_to_f16_kernel(const uint16_t* __restrict__ w, int64_t n,
                       const double* __restrict__ partial, int* __restrict__ e_out,
                       __half* __restrict__ out) {
  __shared__ int se;
  if (threadIdx.x == 0) {
    se = f16_exponent(partial);
    if (blockIdx.x == 0) *e_out = se;
  }
  __syncthreads();
  const int e = se;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * 256)
    out[i] = __double2half(
        ldexp(static_cast<double>(__uint_as_float(static_cast<uint32_t>(w[i]) << 16)), e));
}

// out = a + b elementwise (binary64).
__global__ void add_f64_kernel(const double* __restrict__ a, const double* __restrict__ b,
                               double* __restrict__ out, int64_t n) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    out[i] = __dadd_rn(a[i], b[i]);
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
template <auto kern, size_t kBytes>
cudaError_t gemm_smem_attr() {
  static unsigned long long done = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 64 && (__atomic_load_n(&done, __ATOMIC_ACQUIRE) & (1ull << dev))) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kBytes));
  if (e == cudaSuccess && dev < 64) __atomic_fetch_or(&done, 1ull << dev, __ATOMIC_RELEASE);
  return e;
}

cudaError_t gemm(const GemmArgs& g, bool b_f64, int batch, cudaStream_t st) {
  const dim3 grid(static_cast<unsigned>((g.N + kGN - 1) / kGN),
                  static_cast<unsigned>((g.M + kGM - 1) / kGM), static_cast<unsigned>(batch));
  cudaError_t e;
  if (b_f64) {
    constexpr size_t kBytes = gemm_smem_bytes<double>();
    e = gemm_smem_attr<gemm_f64_kernel<double>, kBytes>();
    if (e != cudaSuccess) return e;
    gemm_f64_kernel<double><<<grid, 256, kBytes, st>>>(g);
  } else {
    // bf16 operands are the linears' weights: k contiguous, K even.
    if (g.sBk != 1 || (g.K & 1) || (g.sBn & 1)) return cudaErrorInvalidValue;
    constexpr size_t kBytes = gemm_smem_bytes<uint16_t>();
    e = gemm_smem_attr<gemm_f64_kernel<uint16_t>, kBytes>();
    if (e != cudaSuccess) return e;
    gemm_f64_kernel<uint16_t><<<grid, 256, kBytes, st>>>(g);
  }
  return cudaGetLastError();
}

// out[T, N] = x[T, K] W^T (+ residual), W row-major [N, K].
cudaError_t linear(const double* x, int T, int K, const void* w, bool w_f64, int N, double* out,
                   const double* residual, cudaStream_t st) {
  GemmArgs g{};
  g.A = x;
  g.sAm = K;
  g.sAk = 1;
  g.B = w;
  g.sBn = K;
  g.sBk = 1;
  g.bdiv = 1;
  g.C = out;
  g.sCm = N;
  g.sCn = 1;
  g.R = residual;
  g.M = T;
  g.N = N;
  g.K = K;
  return gemm(g, w_f64, 1, st);
}

struct Lin {
  const void* p;
  bool f64;
};

// Buffers of one block forward ([T, width] row-major, binary64).
struct Bufs {
  double *h, *q, *k, *v, *S, *a, *x1, *h2, *g, *u, *act;
};

struct Ctx {
  const BlockConfig* c;
  int T;
  cudaStream_t st;
};

cudaError_t run_rmsnorm(const Ctx& cx, const double* x, const double* gamma, double* out) {
  rmsnorm_f64_kernel<<<cx.T, 256, 0, cx.st>>>(x, gamma, cx.c->hidden, cx.c->eps, out);
  return cudaGetLastError();
}

// out = the per-head norm and rotary embedding of in (in == out allowed).
cudaError_t run_qknorm_rope(const Ctx& cx, const double* in, double* out, int heads,
                            const double* gain) {
  const int64_t rows = static_cast<int64_t>(cx.T) * heads;
  const unsigned blocks = static_cast<unsigned>((rows + 7) / 8);
  if (cx.c->head_dim == 128)
    qknorm_rope_kernel<4><<<blocks, 256, 0, cx.st>>>(in, out, rows, heads, gain, cx.c->eps,
                                                     cx.c->rope_theta);
  else
    qknorm_rope_kernel<2><<<blocks, 256, 0, cx.st>>>(in, out, rows, heads, gain, cx.c->eps,
                                                     cx.c->rope_theta);
  return cudaGetLastError();
}

// Block forward from `stage` (0: the q/k/v projections, 1: o, 2: gate/up,
// 3: down).  Buffers before the stage must hold the values of the path
// being continued; b.h must hold RMSNorm(x) for stage 0.  W: q k v o gate
// up down.  out = the block's output.
cudaError_t forward_from(const Ctx& cx, int stage, const double* x, const Lin* W,
                         const BlockNorms& nm, const Bufs& b, double* out) {
  const BlockConfig& c = *cx.c;
  const int T = cx.T, H = c.hidden, d = c.head_dim;
  const int nq = c.heads * d, nkv = c.kv_heads * d, F = c.ffn;
  cudaError_t e = cudaSuccess;
#define W4_TRY(call)               \
  do {                             \
    e = (call);                    \
    if (e != cudaSuccess) return e; \
  } while (0)
  if (stage <= 0) {
    W4_TRY(linear(b.h, T, H, W[0].p, W[0].f64, nq, b.q, nullptr, cx.st));
    W4_TRY(linear(b.h, T, H, W[1].p, W[1].f64, nkv, b.k, nullptr, cx.st));
    W4_TRY(linear(b.h, T, H, W[2].p, W[2].f64, nkv, b.v, nullptr, cx.st));
    W4_TRY(run_qknorm_rope(cx, b.q, b.q, c.heads, nm.q_norm));
    W4_TRY(run_qknorm_rope(cx, b.k, b.k, c.kv_heads, nm.k_norm));
    // S[h] = q_h k_{h/g}^T, causal tiles only.
    GemmArgs g{};
    g.A = b.q;
    g.sAm = nq;
    g.sAk = 1;
    g.bA = d;
    g.B = b.k;
    g.sBn = nkv;
    g.sBk = 1;
    g.bB = d;
    g.bdiv = c.heads / c.kv_heads;
    g.C = b.S;
    g.sCm = T;
    g.sCn = 1;
    g.bC = static_cast<int64_t>(T) * T;
    g.M = T;
    g.N = T;
    g.K = d;
    g.causal = 1;
    W4_TRY(gemm(g, true, c.heads, cx.st));
    const int64_t rows = static_cast<int64_t>(c.heads) * T;
    softmax_causal_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, cx.st>>>(
        b.S, rows, T, sqrt(static_cast<double>(d)));
    W4_TRY(cudaGetLastError());
    // a[t, h, :] = P_h v_{h/g}: B rows are the d channels, k runs over keys.
    GemmArgs p{};
    p.A = b.S;
    p.sAm = T;
    p.sAk = 1;
    p.bA = static_cast<int64_t>(T) * T;
    p.B = b.v;
    p.sBn = 1;
    p.sBk = nkv;
    p.bB = d;
    p.bdiv = c.heads / c.kv_heads;
    p.C = b.a;
    p.sCm = nq;
    p.sCn = 1;
    p.bC = d;
    p.M = T;
    p.N = d;
    p.K = T;
    p.causal = 2;
    W4_TRY(gemm(p, true, c.heads, cx.st));
  }
  if (stage <= 1) {
    W4_TRY(linear(b.a, T, nq, W[3].p, W[3].f64, H, b.x1, x, cx.st));
    W4_TRY(run_rmsnorm(cx, b.x1, nm.ln2, b.h2));
  }
  if (stage <= 2) {
    W4_TRY(linear(b.h2, T, H, W[4].p, W[4].f64, F, b.g, nullptr, cx.st));
    W4_TRY(linear(b.h2, T, H, W[5].p, W[5].f64, F, b.u, nullptr, cx.st));
    const int64_t n = static_cast<int64_t>(T) * F;
    swiglu_f64_kernel<<<592, 256, 0, cx.st>>>(b.g, b.u, b.act, n);
    W4_TRY(cudaGetLastError());
  }
  W4_TRY(linear(b.act, T, F, W[6].p, W[6].f64, H, out, b.x1, cx.st));
#undef W4_TRY
  return cudaSuccess;
}

cudaError_t forward_full(const Ctx& cx, const double* x, const Lin* W, const BlockNorms& nm,
                         const Bufs& b, double* out) {
  cudaError_t e = run_rmsnorm(cx, x, nm.ln1, b.h);
  if (e != cudaSuccess) return e;
  return forward_from(cx, 0, x, W, nm, b, out);
}

// Linears of each group and the width of the group's input.
constexpr int kGroupFirst[5] = {0, 3, 4, 6, 7};

int group_in_width(const BlockConfig& c, int group) {
  switch (group) {
    case 0:
    case 2:
      return c.hidden;
    case 1:
      return c.heads * c.head_dim;
    default:
      return c.ffn;
  }
}

void linear_shape(const BlockConfig& c, int lin, int* n, int* k) {
  const int nq = c.heads * c.head_dim, nkv = c.kv_heads * c.head_dim;
  const int ns[7] = {nq, nkv, nkv, c.hidden, c.ffn, c.ffn, c.hidden};
  const int ks[7] = {c.hidden, c.hidden, c.hidden, nq, c.hidden, c.hidden, c.ffn};
  *n = ns[lin];
  *k = ks[lin];
}

size_t rup(size_t b) { return (b + 255) & ~size_t{255}; }

constexpr int kFBufs = 16;  // buffers of a screening forward (FBufs)

struct Layout {
  size_t bufsA[11], bufsB[11], out_a, out_b, ref, stat, s, wc, partial, loss;
  // Screening: reference and candidate sets of block i and block i+1, the
  // fp16 weights, a candidate's weight change, fp16 operands, exponents.
  size_t fset[4][kFBufs], w16[14], dw64, dw16[3], in16, d16, fpart, exps, floss, total;
};

Layout layout(const BlockConfig& c, int64_t T) {
  const size_t H = c.hidden, nq = static_cast<size_t>(c.heads) * c.head_dim;
  const size_t nkv = static_cast<size_t>(c.kv_heads) * c.head_dim, F = c.ffn;
  const size_t Tz = static_cast<size_t>(T);
  const size_t widths[11] = {H, nq, nkv, nkv, 0, nq, H, H, F, F, F};
  Layout L{};
  size_t off = 0;
  for (int set = 0; set < 2; ++set) {
    size_t* dst = set ? L.bufsB : L.bufsA;
    for (int i = 0; i < 11; ++i) {
      dst[i] = off;
      const size_t elems = i == 4 ? static_cast<size_t>(c.heads) * Tz * Tz : Tz * widths[i];
      off += rup(elems * sizeof(double));
    }
  }
  L.out_a = off;
  off += rup(Tz * H * sizeof(double));
  L.out_b = off;
  off += rup(Tz * H * sizeof(double));
  L.ref = off;
  off += rup(Tz * H * sizeof(double));
  const size_t kmax = std::max(H, std::max(nq, F));
  L.stat = off;
  off += rup(kmax * sizeof(double));
  L.s = off;
  off += rup(kmax * sizeof(float));
  // Candidate weights of the largest group.
  size_t wmax = 0;
  for (int gI = 0; gI < 4; ++gI) {
    size_t sum = 0;
    for (int l = kGroupFirst[gI]; l < kGroupFirst[gI + 1]; ++l) {
      int n, k;
      linear_shape(c, l, &n, &k);
      sum += rup(static_cast<size_t>(n) * k * sizeof(double));
    }
    wmax = std::max(wmax, sum);
  }
  L.wc = off;
  off += wmax;
  L.partial = off;
  off += rup(kLossBlocks * sizeof(double));
  L.loss = off;
  off += rup(2 * kMaxGrid * 11 * sizeof(double));
  // h ql kl v qr kr S a ap x1 h2 g u act mlp out
  const size_t fw[kFBufs] = {H, nq, nkv, nkv, nq, nkv, 0, nq, H, H, H, F, F, F, H, H};
  for (int set = 0; set < 4; ++set)
    for (int i = 0; i < kFBufs; ++i) {
      L.fset[set][i] = off;
      const size_t elems = i == 6 ? static_cast<size_t>(c.heads) * Tz * Tz : Tz * fw[i];
      off += rup(elems * sizeof(double));
    }
  size_t lmax = 0;
  for (int l = 0; l < 14; ++l) {
    int n, k;
    linear_shape(c, l % 7, &n, &k);
    L.w16[l] = off;
    off += rup(static_cast<size_t>(n) * k * 2);
    lmax = std::max(lmax, static_cast<size_t>(n) * k);
  }
  L.dw64 = off;
  off += rup(lmax * sizeof(double));
  for (int i = 0; i < 3; ++i) {
    L.dw16[i] = off;
    off += rup(lmax * 2);
  }
  L.in16 = off;
  off += rup(Tz * kmax * 2);
  L.d16 = off;
  off += rup(Tz * kmax * 2);
  L.fpart = off;
  off += rup(kLossBlocks * sizeof(double));
  L.exps = off;
  off += rup(64 * sizeof(int));
  L.floss = off;
  off += rup(kMaxGrid * sizeof(double));
  L.total = off;
  return L;
}

Bufs bufs_at(uint8_t* ws, const size_t* off) {
  double* p[11];
  for (int i = 0; i < 11; ++i) p[i] = reinterpret_cast<double*>(ws + off[i]);
  return Bufs{p[0], p[1], p[2], p[3], p[4], p[5], p[6], p[7], p[8], p[9], p[10]};
}

struct Session {
  Ctx cx;
  const BlockConfig* c;
  const double* x;
  Lin Wi[7], Wn[7];
  BlockNorms ni, nn;
  bool ahead;
  Bufs A, B;
  uint8_t* ws;
  Layout L;
  bool sym;
  AlphaList al;
  ShrinkList sl;
  unsigned* err;  // device error word (tcgen05 waits)
};

Session make_session(const BlockConfig* c, const double* x, int64_t T, const BlockLinears& blk,
                     const BlockLinears* next, const float* alphas, int n_alpha,
                     const float* shrinks, int n_shrink, bool sym, void* workspace,
                     cudaStream_t st) {
  Session s{};
  s.cx = Ctx{c, static_cast<int>(T), st};
  s.c = c;
  s.x = x;
  for (int i = 0; i < 7; ++i) s.Wi[i] = Lin{blk.w[i], false};
  s.ni = blk.norms;
  s.ahead = next != nullptr;
  if (next) {
    for (int i = 0; i < 7; ++i) s.Wn[i] = Lin{next->w[i], false};
    s.nn = next->norms;
  }
  s.ws = static_cast<uint8_t*>(workspace);
  s.L = layout(*c, T);
  s.A = bufs_at(s.ws, s.L.bufsA);
  s.B = bufs_at(s.ws, s.L.bufsB);
  s.sym = sym;
  s.al.n = n_alpha;
  for (int i = 0; i < n_alpha; ++i) s.al.v[i] = alphas[i];
  s.sl.n = n_shrink;
  for (int j = 0; j < n_shrink; ++j) s.sl.v[j] = shrinks[j];
  return s;
}

double* ws_d(const Session& s, size_t off) { return reinterpret_cast<double*>(s.ws + off); }

// The unquantized path: block i (its intermediates stay in set A), block
// i+1 on it if scored ahead; ref = the path's output; stat = the group's
// AWQ statistic.
cudaError_t reference(const Session& s, int group) {
  double* out_i = ws_d(s, s.L.out_a);
  cudaError_t e = forward_full(s.cx, s.x, s.Wi, s.ni, s.A, out_i);
  if (e != cudaSuccess) return e;
  double* ref = ws_d(s, s.L.ref);
  if (s.ahead) {
    e = forward_full(s.cx, out_i, s.Wn, s.nn, s.B, ref);
  } else {
    e = cudaMemcpyAsync(ref, out_i, sizeof(double) * s.cx.T * s.c->hidden,
                        cudaMemcpyDeviceToDevice, s.cx.st);
  }
  if (e != cudaSuccess) return e;
  const double* in[4] = {s.A.h, s.A.a, s.A.h2, s.A.act};
  const int K = group_in_width(*s.c, group);
  colmean_abs_f64_kernel<<<(K + 127) / 128, 128, 0, s.cx.st>>>(in[group], s.cx.T, K,
                                                               ws_d(s, s.L.stat));
  return cudaGetLastError();
}

// Loss of one candidate of `group`: alpha alphas[ia] (or alphas[*ia_dev]),
// shrink `ratio` on linear `only` (every linear of the group if only < 0),
// the group's other linears unclipped.  loss_out: device double.
cudaError_t candidate(const Session& s, int group, int ia, const int32_t* ia_dev, float ratio,
                      int only, double* loss_out) {
  const BlockConfig& c = *s.c;
  const int K = group_in_width(c, group);
  float* sv = reinterpret_cast<float*>(s.ws + s.L.s);
  block_scales_kernel<<<(K + 127) / 128, 128, 0, s.cx.st>>>(ws_d(s, s.L.stat), K, s.al, ia,
                                                            ia_dev, sv);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  Lin W[7];
  for (int i = 0; i < 7; ++i) W[i] = s.Wi[i];
  size_t off = s.L.wc;
  for (int l = kGroupFirst[group]; l < kGroupFirst[group + 1]; ++l) {
    int n, k;
    linear_shape(c, l, &n, &k);
    double* wc = ws_d(s, off);
    off += rup(static_cast<size_t>(n) * k * sizeof(double));
    const float r = (only < 0 || only == l) ? ratio : 1.0f;
    const int64_t items = static_cast<int64_t>(n) * (k / 128);
    const unsigned blocks = static_cast<unsigned>((items + 7) / 8);
    const auto* wb = static_cast<const uint16_t*>(s.Wi[l].p);
    if (s.sym)
      candidate_weight_kernel<true><<<blocks, 256, 0, s.cx.st>>>(wb, n, k, sv, r, wc);
    else
      candidate_weight_kernel<false><<<blocks, 256, 0, s.cx.st>>>(wb, n, k, sv, r, wc);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    W[l] = Lin{wc, true};
  }
  double* out_i = ws_d(s, s.L.out_b);
  e = forward_from(s.cx, group, s.x, W, s.ni, s.A, out_i);
  if (e != cudaSuccess) return e;
  const double* fin = out_i;
  if (s.ahead) {
    double* out_n = ws_d(s, s.L.out_a);  // the reference's block-i output is no longer needed
    e = forward_full(s.cx, out_i, s.Wn, s.nn, s.B, out_n);
    if (e != cudaSuccess) return e;
    fin = out_n;
  }
  const int64_t n = static_cast<int64_t>(s.cx.T) * c.hidden;
  double* part = ws_d(s, s.L.partial);
  sqdiff_partial_kernel<<<kLossBlocks, 256, 0, s.cx.st>>>(fin, ws_d(s, s.L.ref), n, part);
  loss_finish_kernel<<<1, 32, 0, s.cx.st>>>(part, n, loss_out);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Screening forward.  The reference path keeps every intermediate in
// binary64.  A candidate's path is then the reference plus its change: each
// linear after the group is y_ref + (x - x_ref) W^T and each linear of the
// group y_ref + x_ref (W_c - W)^T, the products on the tcgen05 tensor cores
// with fp16 operands scaled by exact powers of two and binary64 epilogues;
// norms, rotary embedding, attention and SwiGLU run in binary64 on the full
// values.  The products round only the changes (about 2^-11 of each), so the
// losses are close to the binary64 ones; selections decide their near ties
// on the binary64 path.
// ---------------------------------------------------------------------------
struct FBufs {
  double *h, *ql, *kl, *v, *qr, *kr, *S, *a, *ap, *x1, *h2, *g, *u, *act, *mlp, *out;
};

FBufs fbufs_at(uint8_t* ws, const size_t* off) {
  double* p[kFBufs];
  for (int i = 0; i < kFBufs; ++i) p[i] = reinterpret_cast<double*>(ws + off[i]);
  return FBufs{p[0], p[1], p[2], p[3], p[4], p[5], p[6], p[7],
               p[8], p[9], p[10], p[11], p[12], p[13], p[14], p[15]};
}

// Exponent slots: 0..6 block i's weights, 7..13 block i+1's, 14..16 the
// group's weight changes, 17 the group's input, 18 the current change.
constexpr int kSlotDw = 14, kSlotIn = 17, kSlotD = 18;

#define W4_TRY(call)               \
  do {                             \
    cudaError_t e_ = (call);       \
    if (e_ != cudaSuccess) return e_; \
  } while (0)

cudaError_t run_add(const Ctx& cx, const double* a, const double* b, double* out, int64_t n) {
  add_f64_kernel<<<592, 256, 0, cx.st>>>(a, b, out, n);
  return cudaGetLastError();
}

// q, k (after their norms and rotary embedding) and v -> S -> P -> a.
cudaError_t attention(const Ctx& cx, const double* q, const double* k, const double* v, double* S,
                      double* a) {
  const BlockConfig& c = *cx.c;
  const int T = cx.T, d = c.head_dim;
  const int nq = c.heads * d, nkv = c.kv_heads * d;
  GemmArgs g{};
  g.A = q;
  g.sAm = nq;
  g.sAk = 1;
  g.bA = d;
  g.B = k;
  g.sBn = nkv;
  g.sBk = 1;
  g.bB = d;
  g.bdiv = c.heads / c.kv_heads;
  g.C = S;
  g.sCm = T;
  g.sCn = 1;
  g.bC = static_cast<int64_t>(T) * T;
  g.M = T;
  g.N = T;
  g.K = d;
  g.causal = 1;
  W4_TRY(gemm(g, true, c.heads, cx.st));
  const int64_t rows = static_cast<int64_t>(c.heads) * T;
  softmax_causal_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, cx.st>>>(
      S, rows, T, sqrt(static_cast<double>(d)));
  W4_TRY(cudaGetLastError());
  GemmArgs p{};
  p.A = S;
  p.sAm = T;
  p.sAk = 1;
  p.bA = static_cast<int64_t>(T) * T;
  p.B = v;
  p.sBn = 1;
  p.sBk = nkv;
  p.bB = d;
  p.bdiv = c.heads / c.kv_heads;
  p.C = a;
  p.sCm = nq;
  p.sCn = 1;
  p.bC = d;
  p.M = T;
  p.N = d;
  p.K = T;
  p.causal = 2;
  return gemm(p, true, c.heads, cx.st);
}

// The reference path of one block with every intermediate kept (binary64;
// the same kernels and order as forward_from, so the values are those of
// the binary64 path).
cudaError_t fwd_ref(const Ctx& cx, const double* x, const Lin* W, const BlockNorms& nm,
                    const FBufs& R) {
  const BlockConfig& c = *cx.c;
  const int T = cx.T, H = c.hidden, nq = c.heads * c.head_dim, nkv = c.kv_heads * c.head_dim;
  const int F = c.ffn;
  const int64_t th = static_cast<int64_t>(T) * H;
  W4_TRY(run_rmsnorm(cx, x, nm.ln1, R.h));
  W4_TRY(linear(R.h, T, H, W[0].p, W[0].f64, nq, R.ql, nullptr, cx.st));
  W4_TRY(linear(R.h, T, H, W[1].p, W[1].f64, nkv, R.kl, nullptr, cx.st));
  W4_TRY(linear(R.h, T, H, W[2].p, W[2].f64, nkv, R.v, nullptr, cx.st));
  W4_TRY(run_qknorm_rope(cx, R.ql, R.qr, c.heads, nm.q_norm));
  W4_TRY(run_qknorm_rope(cx, R.kl, R.kr, c.kv_heads, nm.k_norm));
  W4_TRY(attention(cx, R.qr, R.kr, R.v, R.S, R.a));
  W4_TRY(linear(R.a, T, nq, W[3].p, W[3].f64, H, R.ap, nullptr, cx.st));
  W4_TRY(run_add(cx, x, R.ap, R.x1, th));
  W4_TRY(run_rmsnorm(cx, R.x1, nm.ln2, R.h2));
  W4_TRY(linear(R.h2, T, H, W[4].p, W[4].f64, F, R.g, nullptr, cx.st));
  W4_TRY(linear(R.h2, T, H, W[5].p, W[5].f64, F, R.u, nullptr, cx.st));
  swiglu_f64_kernel<<<592, 256, 0, cx.st>>>(R.g, R.u, R.act, static_cast<int64_t>(T) * F);
  W4_TRY(cudaGetLastError());
  W4_TRY(linear(R.act, T, F, W[6].p, W[6].f64, H, R.mlp, nullptr, cx.st));
  return run_add(cx, R.x1, R.mlp, R.out, th);
}

struct Screen {
  const Session* s;
  FBufs Ri, Rn, Ci, Cn;
  __half* w16[14];
  __half* dw16[3];
  double* dw64;
  __half* in16;
  __half* d16;
  double* part;
  int* exps;
  double* floss;
};

Screen make_screen(const Session& s) {
  Screen z{};
  z.s = &s;
  z.Ri = fbufs_at(s.ws, s.L.fset[0]);
  z.Rn = fbufs_at(s.ws, s.L.fset[1]);
  z.Ci = fbufs_at(s.ws, s.L.fset[2]);
  z.Cn = fbufs_at(s.ws, s.L.fset[3]);
  for (int l = 0; l < 14; ++l) z.w16[l] = reinterpret_cast<__half*>(s.ws + s.L.w16[l]);
  for (int i = 0; i < 3; ++i) z.dw16[i] = reinterpret_cast<__half*>(s.ws + s.L.dw16[i]);
  z.dw64 = reinterpret_cast<double*>(s.ws + s.L.dw64);
  z.in16 = reinterpret_cast<__half*>(s.ws + s.L.in16);
  z.d16 = reinterpret_cast<__half*>(s.ws + s.L.d16);
  z.part = reinterpret_cast<double*>(s.ws + s.L.fpart);
  z.exps = reinterpret_cast<int*>(s.ws + s.L.exps);
  z.floss = reinterpret_cast<double*>(s.ws + s.L.floss);
  return z;
}

// out = fp16((a - b) 2^e), exps[slot] = e (b may be null).
cudaError_t to_f16(const Screen& z, const double* a, const double* b, int64_t n, int slot,
                   __half* out) {
  const cudaStream_t st = z.s->cx.st;
  absmax_partial_kernel<<<kLossBlocks, 256, 0, st>>>(a, b, n, z.part);
  to_f16_kernel<<<592, 256, 0, st>>>(a, b, n, z.part, z.exps + slot, out);
  return cudaGetLastError();
}

// out[T, N] = r1 (+ r2) + A B^T with A = fp16 operand of slot sa, B of slot sb.
cudaError_t add_gemm(const Screen& z, const __half* a16, int sa, const __half* b16, int sb, int N,
                     int K, double* out, const double* r1, const double* r2) {
  return launch_add_gemm_f16(a16, z.s->cx.T, b16, N, K, out, N, r1, r2, z.exps + sa, z.exps + sb,
                             z.s->cx.st, z.s->err);
}

// The reference paths and the fp16 weights of both blocks.
cudaError_t screen_prepare(const Screen& z) {
  const Session& s = *z.s;
  const cudaStream_t st = s.cx.st;
  for (int l = 0; l < (s.ahead ? 14 : 7); ++l) {
    int n, k;
    linear_shape(*s.c, l % 7, &n, &k);
    const int64_t nk = static_cast<int64_t>(n) * k;
    const auto* w = static_cast<const uint16_t*>(l < 7 ? s.Wi[l].p : s.Wn[l - 7].p);
    absmax_partial_bf16_kernel<<<kLossBlocks, 256, 0, st>>>(w, nk, z.part);
    bf16_to_f16_kernel<<<592, 256, 0, st>>>(w, nk, z.part, z.exps + l, z.w16[l]);
    W4_TRY(cudaGetLastError());
  }
  W4_TRY(fwd_ref(s.cx, s.x, s.Wi, s.ni, z.Ri));
  if (s.ahead) W4_TRY(fwd_ref(s.cx, z.Ri.out, s.Wn, s.nn, z.Rn));
  return cudaSuccess;
}

// A group's statistic and its input in fp16 (slot kSlotIn).
cudaError_t screen_group(const Screen& z, int group) {
  const Session& s = *z.s;
  const double* in[4] = {z.Ri.h, z.Ri.a, z.Ri.h2, z.Ri.act};
  const int K = group_in_width(*s.c, group);
  colmean_abs_f64_kernel<<<(K + 127) / 128, 128, 0, s.cx.st>>>(in[group], s.cx.T, K,
                                                               ws_d(s, s.L.stat));
  W4_TRY(cudaGetLastError());
  return to_f16(z, in[group], nullptr, static_cast<int64_t>(s.cx.T) * K, kSlotIn, z.in16);
}

// Screening loss of one candidate (alpha index ia, ratio on linear `only`
// or on every linear of the group) into loss_out (device).
cudaError_t screen_candidate(const Screen& z, int group, int ia, float ratio, int only,
                             double* loss_out) {
  const Session& s = *z.s;
  const BlockConfig& c = *s.c;
  const cudaStream_t st = s.cx.st;
  const int T = s.cx.T, H = c.hidden, nq = c.heads * c.head_dim, nkv = c.kv_heads * c.head_dim;
  const int F = c.ffn;
  const int64_t th = static_cast<int64_t>(T) * H;
  const int K = group_in_width(c, group);
  float* sv = reinterpret_cast<float*>(s.ws + s.L.s);
  block_scales_kernel<<<(K + 127) / 128, 128, 0, st>>>(ws_d(s, s.L.stat), K, s.al, ia, nullptr,
                                                       sv);
  W4_TRY(cudaGetLastError());
  // The group's weight changes, fp16 (slots kSlotDw + i).
  for (int l = kGroupFirst[group]; l < kGroupFirst[group + 1]; ++l) {
    int n, k;
    linear_shape(c, l, &n, &k);
    const float r = (only < 0 || only == l) ? ratio : 1.0f;
    const int64_t items = static_cast<int64_t>(n) * (k / 128);
    const unsigned blocks = static_cast<unsigned>((items + 7) / 8);
    const auto* wb = static_cast<const uint16_t*>(s.Wi[l].p);
    if (s.sym)
      candidate_weight_kernel<true, true><<<blocks, 256, 0, st>>>(wb, n, k, sv, r, z.dw64);
    else
      candidate_weight_kernel<false, true><<<blocks, 256, 0, st>>>(wb, n, k, sv, r, z.dw64);
    W4_TRY(cudaGetLastError());
    const int i = l - kGroupFirst[group];
    W4_TRY(to_f16(z, z.dw64, nullptr, static_cast<int64_t>(n) * k, kSlotDw + i, z.dw16[i]));
  }
  const FBufs &R = z.Ri, &C = z.Ci;
  // Block i from the group on.
  if (group == 0) {
    W4_TRY(add_gemm(z, z.in16, kSlotIn, z.dw16[0], kSlotDw + 0, nq, H, C.ql, R.ql, nullptr));
    W4_TRY(add_gemm(z, z.in16, kSlotIn, z.dw16[1], kSlotDw + 1, nkv, H, C.kl, R.kl, nullptr));
    W4_TRY(add_gemm(z, z.in16, kSlotIn, z.dw16[2], kSlotDw + 2, nkv, H, C.v, R.v, nullptr));
    W4_TRY(run_qknorm_rope(s.cx, C.ql, C.qr, c.heads, s.ni.q_norm));
    W4_TRY(run_qknorm_rope(s.cx, C.kl, C.kr, c.kv_heads, s.ni.k_norm));
    W4_TRY(attention(s.cx, C.qr, C.kr, C.v, C.S, C.a));
    W4_TRY(to_f16(z, C.a, R.a, static_cast<int64_t>(T) * nq, kSlotD, z.d16));
    W4_TRY(add_gemm(z, z.d16, kSlotD, z.w16[3], 3, H, nq, C.x1, s.x, R.ap));
  } else if (group == 1) {
    W4_TRY(add_gemm(z, z.in16, kSlotIn, z.dw16[0], kSlotDw, H, nq, C.x1, R.x1, nullptr));
  }
  if (group <= 1) {
    W4_TRY(run_rmsnorm(s.cx, C.x1, s.ni.ln2, C.h2));
    W4_TRY(to_f16(z, C.h2, R.h2, th, kSlotD, z.d16));
    W4_TRY(add_gemm(z, z.d16, kSlotD, z.w16[4], 4, F, H, C.g, R.g, nullptr));
    W4_TRY(add_gemm(z, z.d16, kSlotD, z.w16[5], 5, F, H, C.u, R.u, nullptr));
  } else if (group == 2) {
    W4_TRY(add_gemm(z, z.in16, kSlotIn, z.dw16[0], kSlotDw + 0, F, H, C.g, R.g, nullptr));
    W4_TRY(add_gemm(z, z.in16, kSlotIn, z.dw16[1], kSlotDw + 1, F, H, C.u, R.u, nullptr));
  }
  if (group <= 2) {
    swiglu_f64_kernel<<<592, 256, 0, st>>>(C.g, C.u, C.act, static_cast<int64_t>(T) * F);
    W4_TRY(cudaGetLastError());
    W4_TRY(to_f16(z, C.act, R.act, static_cast<int64_t>(T) * F, kSlotD, z.d16));
    W4_TRY(add_gemm(z, z.d16, kSlotD, z.w16[6], 6, H, F, C.out, group <= 1 ? C.x1 : R.x1,
                    R.mlp));
  } else {
    W4_TRY(add_gemm(z, z.in16, kSlotIn, z.dw16[0], kSlotDw, H, F, C.out, R.out, nullptr));
  }
  const double* fin = C.out;
  const double* ref = R.out;
  if (s.ahead) {
    // Block i+1 on the changed input: every linear is y_ref + change.
    const FBufs &Rn = z.Rn, &Cn = z.Cn;
    W4_TRY(run_rmsnorm(s.cx, C.out, s.nn.ln1, Cn.h));
    W4_TRY(to_f16(z, Cn.h, Rn.h, th, kSlotD, z.d16));
    W4_TRY(add_gemm(z, z.d16, kSlotD, z.w16[7], 7, nq, H, Cn.ql, Rn.ql, nullptr));
    W4_TRY(add_gemm(z, z.d16, kSlotD, z.w16[8], 8, nkv, H, Cn.kl, Rn.kl, nullptr));
    W4_TRY(add_gemm(z, z.d16, kSlotD, z.w16[9], 9, nkv, H, Cn.v, Rn.v, nullptr));
    W4_TRY(run_qknorm_rope(s.cx, Cn.ql, Cn.qr, c.heads, s.nn.q_norm));
    W4_TRY(run_qknorm_rope(s.cx, Cn.kl, Cn.kr, c.kv_heads, s.nn.k_norm));
    W4_TRY(attention(s.cx, Cn.qr, Cn.kr, Cn.v, Cn.S, Cn.a));
    W4_TRY(to_f16(z, Cn.a, Rn.a, static_cast<int64_t>(T) * nq, kSlotD, z.d16));
    W4_TRY(add_gemm(z, z.d16, kSlotD, z.w16[10], 10, H, nq, Cn.x1, C.out, Rn.ap));
    W4_TRY(run_rmsnorm(s.cx, Cn.x1, s.nn.ln2, Cn.h2));
    W4_TRY(to_f16(z, Cn.h2, Rn.h2, th, kSlotD, z.d16));
    W4_TRY(add_gemm(z, z.d16, kSlotD, z.w16[11], 11, F, H, Cn.g, Rn.g, nullptr));
    W4_TRY(add_gemm(z, z.d16, kSlotD, z.w16[12], 12, F, H, Cn.u, Rn.u, nullptr));
    swiglu_f64_kernel<<<592, 256, 0, st>>>(Cn.g, Cn.u, Cn.act, static_cast<int64_t>(T) * F);
    W4_TRY(cudaGetLastError());
    W4_TRY(to_f16(z, Cn.act, Rn.act, static_cast<int64_t>(T) * F, kSlotD, z.d16));
    W4_TRY(add_gemm(z, z.d16, kSlotD, z.w16[13], 13, H, F, Cn.out, Cn.x1, Rn.mlp));
    fin = Cn.out;
    ref = Rn.out;
  }
  double* part = ws_d(s, s.L.partial);
  sqdiff_partial_kernel<<<kLossBlocks, 256, 0, st>>>(fin, ref, th, part);
  loss_finish_kernel<<<1, 32, 0, st>>>(part, th, loss_out);
  return cudaGetLastError();
}

// The binary64 loss of one candidate for a screened selection: the same
// path as candidate(), reading the group's inputs (and the residuals before
// the group) from the screening's reference set, which holds the binary64
// reference values (fwd_ref runs forward_from's kernels in its order), and
// writing everything from the group on into set A / set B.
cudaError_t exact_candidate(const Screen& z, int group, int ia, float ratio, int only,
                            double* loss_out) {
  const Session& s = *z.s;
  const BlockConfig& c = *s.c;
  const cudaStream_t st = s.cx.st;
  const int K = group_in_width(c, group);
  float* sv = reinterpret_cast<float*>(s.ws + s.L.s);
  block_scales_kernel<<<(K + 127) / 128, 128, 0, st>>>(ws_d(s, s.L.stat), K, s.al, ia, nullptr,
                                                       sv);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  Lin W[7];
  for (int i = 0; i < 7; ++i) W[i] = s.Wi[i];
  size_t off = s.L.wc;
  for (int l = kGroupFirst[group]; l < kGroupFirst[group + 1]; ++l) {
    int n, k;
    linear_shape(c, l, &n, &k);
    double* wc = ws_d(s, off);
    off += rup(static_cast<size_t>(n) * k * sizeof(double));
    const float r = (only < 0 || only == l) ? ratio : 1.0f;
    const int64_t items = static_cast<int64_t>(n) * (k / 128);
    const unsigned blocks = static_cast<unsigned>((items + 7) / 8);
    const auto* wb = static_cast<const uint16_t*>(s.Wi[l].p);
    if (s.sym)
      candidate_weight_kernel<true><<<blocks, 256, 0, st>>>(wb, n, k, sv, r, wc);
    else
      candidate_weight_kernel<false><<<blocks, 256, 0, st>>>(wb, n, k, sv, r, wc);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    W[l] = Lin{wc, true};
  }
  // Inputs before the group from the reference set, the rest into set A.
  const FBufs& R = z.Ri;
  Bufs b = s.A;
  b.h = R.h;
  if (group >= 1) b.a = R.a;
  if (group >= 2) {
    b.x1 = R.x1;
    b.h2 = R.h2;
  }
  if (group >= 3) b.act = R.act;
  double* out_i = ws_d(s, s.L.out_b);
  e = forward_from(s.cx, group, s.x, W, s.ni, b, out_i);
  if (e != cudaSuccess) return e;
  const double* fin = out_i;
  const double* ref = R.out;
  if (s.ahead) {
    double* out_n = ws_d(s, s.L.out_a);
    e = forward_full(s.cx, out_i, s.Wn, s.nn, s.B, out_n);
    if (e != cudaSuccess) return e;
    fin = out_n;
    ref = z.Rn.out;
  }
  const int64_t n = static_cast<int64_t>(s.cx.T) * c.hidden;
  double* part = ws_d(s, s.L.partial);
  sqdiff_partial_kernel<<<kLossBlocks, 256, 0, st>>>(fin, ref, n, part);
  loss_finish_kernel<<<1, 32, 0, st>>>(part, n, loss_out);
  return cudaGetLastError();
}

__global__ void set_int_kernel(int32_t* p, int v) {
  if (threadIdx.x == 0) *p = v;
}

// One selection of the search: screening losses of n candidates (cand(i)
// = alpha index, ratio), near ties decided on the binary64 path.  Returns
// the chosen index in *pick; losses (device, n) receive the values used.
template <typename CandFn>
cudaError_t screened_select(const Screen& z, int group, int n, int only, CandFn cand,
                            double* losses, int* pick) {
  const Session& s = *z.s;
  for (int i = 0; i < n; ++i) {
    int ia;
    float r;
    cand(i, &ia, &r);
    W4_TRY(screen_candidate(z, group, ia, r, only, losses + i));
  }
  double host[kMaxGrid];
  W4_TRY(cudaMemcpyAsync(host, losses, sizeof(double) * n, cudaMemcpyDeviceToHost, s.cx.st));
  W4_TRY(cudaStreamSynchronize(s.cx.st));
  double mn = host[0];
  for (int i = 1; i < n; ++i) mn = fmin(mn, host[i]);
  int members = 0;
  bool near[kMaxGrid];
  for (int i = 0; i < n; ++i) {
    near[i] = host[i] <= mn * (1.0 + kBlockTieTol);
    members += near[i];
  }
  if (members >= 2) {
    // Binary64 losses of the near set.
    for (int i = 0; i < n; ++i)
      if (near[i]) {
        int ia;
        float r;
        cand(i, &ia, &r);
        W4_TRY(exact_candidate(z, group, ia, r, only, losses + i));
      }
    W4_TRY(cudaMemcpyAsync(host, losses, sizeof(double) * n, cudaMemcpyDeviceToHost, s.cx.st));
    W4_TRY(cudaStreamSynchronize(s.cx.st));
  }
  int best = -1;
  for (int i = 0; i < n; ++i)
    if (near[i] && (best < 0 || host[i] < host[best])) best = i;
  *pick = best;
  return cudaSuccess;
}

#undef W4_TRY

}  // namespace

size_t block_workspace_bytes(const BlockConfig& c, int64_t T) { return layout(c, T).total; }

cudaError_t block_scoring_losses(const BlockConfig* c, const double* x, int64_t T,
                                 const BlockLinears& blk, const BlockLinears* next, int group,
                                 const float* alphas, int n_alpha, const float* shrinks,
                                 int n_shrink, bool sym, int only, double* losses,
                                 void* workspace, cudaStream_t st) {
  Session s = make_session(c, x, T, blk, next, alphas, n_alpha, shrinks, n_shrink, sym,
                           workspace, st);
  cudaError_t e = reference(s, group);
  if (e != cudaSuccess) return e;
  for (int a = 0; a < n_alpha; ++a)
    for (int j = 0; j < n_shrink; ++j) {
      e = candidate(s, group, a, nullptr, shrinks[j], only, losses + a * n_shrink + j);
      if (e != cudaSuccess) return e;
    }
  return cudaSuccess;
}

cudaError_t block_search(const BlockConfig* c, const double* x, int64_t T, const BlockLinears& blk,
                         const BlockLinears* next, const float* alphas, int n_alpha,
                         const float* shrinks, int n_shrink, bool sym, int32_t* choice,
                         double* losses, void* workspace, cudaStream_t st, unsigned* err) {
  Session s = make_session(c, x, T, blk, next, alphas, n_alpha, shrinks, n_shrink, sym,
                           workspace, st);
  s.err = err;
  const Screen z = make_screen(s);
  double* lbuf = losses ? losses : ws_d(s, s.L.loss);
  double* alpha_l = lbuf;                 // [4][n_alpha]
  double* shrink_l = lbuf + 4 * n_alpha;  // [7][n_shrink]
  cudaError_t e = screen_prepare(z);
  if (e != cudaSuccess) return e;
  for (int group = 0; group < 4; ++group) {
    e = screen_group(z, group);
    if (e != cudaSuccess) return e;
    int a_star = 0;
    e = screened_select(
        z, group, n_alpha, -1,
        [&](int i, int* ia, float* r) {
          *ia = i;
          *r = 1.0f;
        },
        alpha_l + group * n_alpha, &a_star);
    if (e != cudaSuccess) return e;
    set_int_kernel<<<1, 32, 0, st>>>(choice + group, a_star);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    for (int l = kGroupFirst[group]; l < kGroupFirst[group + 1]; ++l) {
      int r_star = 0;
      e = screened_select(
          z, group, n_shrink, l,
          [&](int i, int* ia, float* r) {
            *ia = a_star;
            *r = shrinks[i];
          },
          shrink_l + l * n_shrink, &r_star);
      if (e != cudaSuccess) return e;
      set_int_kernel<<<1, 32, 0, st>>>(choice + 4 + l, r_star);
      e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
  }
  return cudaSuccess;
}

}  // namespace w4
