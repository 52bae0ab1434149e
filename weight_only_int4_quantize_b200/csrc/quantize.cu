// Quantize + pack kernel: bf16 weight [N, K] -> int32 codes [N, K/8],
// fp16 scales [N, K/128], fp16 zeros [N, K/128] (asymmetric).
//
// HBM-bound: 2 bytes read and 0.5 + 4/128 (asymmetric) bytes written per
// weight.  The weight is a sequence of N*K/128 contiguous 256-byte groups;
// each half warp owns one group per step, each lane one 16-byte vector of 8
// values, so loads are fully coalesced 16-byte vectors and the 16 packed
// words of a group are one contiguous 64-byte store.  Group min/max use
// half-warp shuffles; codes use the division-free exact rounding of
// quant_group.cuh.
#include "quant_group.cuh"
#include "w4_kernels.h"

namespace w4 {

namespace {

constexpr int kQuantThreads = 256;
constexpr int kQuantUnroll = 4;  // groups in flight per half warp

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

template <bool SYM, bool HAS_S>
__global__ void __launch_bounds__(kQuantThreads)
    quantize_pack_kernel(const uint4* __restrict__ w, const float* __restrict__ s, float shrink,
                         int64_t n_groups, int64_t groups_per_row, uint32_t* __restrict__ qw,
                         uint16_t* __restrict__ scales, uint16_t* __restrict__ zeros) {
  const int lane = threadIdx.x & 31;
  const int half = lane >> 4;
  const int l16 = lane & 15;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kQuantThreads + threadIdx.x) >> 5;
  const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * kQuantThreads) >> 5;
  // Warp unit u covers groups 2u and 2u+1; the loop bound is warp-uniform.
  const int64_t n_units = (n_groups + 1) >> 1;

  for (int64_t u0 = warp; u0 < n_units; u0 += n_warps * kQuantUnroll) {
    uint4 raw[kQuantUnroll];
    int64_t gi[kQuantUnroll];
#pragma unroll
    for (int i = 0; i < kQuantUnroll; ++i) {
      gi[i] = 2 * (u0 + i * n_warps) + half;
      raw[i] = make_uint4(0, 0, 0, 0);
      if (gi[i] < n_groups) raw[i] = ld_stream(w + gi[i] * 16 + l16);
    }
#pragma unroll
    for (int i = 0; i < kQuantUnroll; ++i) {
      if (u0 + i * n_warps >= n_units) break;  // warp-uniform
      float v[8];
      bf16x8_to_f32(raw[i], v);
      if (HAS_S) {
        const int64_t k0 = (gi[i] % groups_per_row) * 128 + l16 * 8;
        const float4 s0 = __ldg(reinterpret_cast<const float4*>(s + k0));
        const float4 s1 = __ldg(reinterpret_cast<const float4*>(s + k0 + 4));
        v[0] = __fmul_rn(v[0], s0.x); v[1] = __fmul_rn(v[1], s0.y);
        v[2] = __fmul_rn(v[2], s0.z); v[3] = __fmul_rn(v[3], s0.w);
        v[4] = __fmul_rn(v[4], s1.x); v[5] = __fmul_rn(v[5], s1.y);
        v[6] = __fmul_rn(v[6], s1.z); v[7] = __fmul_rn(v[7], s1.w);
      }
      GroupQ g;
      if (SYM) {
        float a = fabsf(v[0]);
#pragma unroll
        for (int j = 1; j < 8; ++j) a = fmaxf(a, fabsf(v[j]));
        g = group_params<true>(hw_max(a), 0.f, shrink);
      } else {
        float mx = v[0], mn = v[0];
#pragma unroll
        for (int j = 1; j < 8; ++j) { mx = fmaxf(mx, v[j]); mn = fminf(mn, v[j]); }
        g = group_params<false>(hw_max(mx), hw_min(mn), shrink);
      }
      uint32_t word = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) word |= code_of(v[j], g) << (4 * nibble_pos(j));
      if (gi[i] < n_groups) {
        qw[gi[i] * 16 + l16] = word;
        if (l16 == 0) {
          scales[gi[i]] = g.s16;
          if (!SYM) zeros[gi[i]] = g.z16;
        }
      }
    }
  }
}

}  // namespace

cudaError_t launch_quantize_pack(const void* w, int64_t N, int64_t K, bool symmetric,
                                 const float* s, float shrink, int32_t* qweight, uint16_t* scales,
                                 uint16_t* zeros, cudaStream_t stream, int num_sms) {
  const int64_t n_groups = N * (K / 128);
  const int64_t n_units = (n_groups + 1) / 2;
  const int64_t warps_needed = (n_units + kQuantUnroll - 1) / kQuantUnroll;
  int64_t blocks = (warps_needed + (kQuantThreads / 32) - 1) / (kQuantThreads / 32);
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;  // 8 x 256 threads per SM
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  const uint4* wp = static_cast<const uint4*>(w);
  uint32_t* qp = reinterpret_cast<uint32_t*>(qweight);
  const int64_t gpr = K / 128;
  dim3 grid(static_cast<unsigned>(blocks)), block(kQuantThreads);
  if (symmetric) {
    if (s) quantize_pack_kernel<true, true><<<grid, block, 0, stream>>>(wp, s, shrink, n_groups, gpr, qp, scales, zeros);
    else   quantize_pack_kernel<true, false><<<grid, block, 0, stream>>>(wp, s, shrink, n_groups, gpr, qp, scales, zeros);
  } else {
    if (s) quantize_pack_kernel<false, true><<<grid, block, 0, stream>>>(wp, s, shrink, n_groups, gpr, qp, scales, zeros);
    else   quantize_pack_kernel<false, false><<<grid, block, 0, stream>>>(wp, s, shrink, n_groups, gpr, qp, scales, zeros);
  }
  return cudaGetLastError();
}

}  // namespace w4
