// Per-token symmetric int8 activations for the W4A8 decode path
// ("malaiwah/GLM-5.2-QSRT-Fruit-Instruct" card: W4A8 decode execution over
// the same stored weights, for decode-sized batches of at most 16 rows).
//
// For token row m:  scale_m = max_k |x_mk| / 127 (binary32),
//                   q_mk = clamp(rint(x_mk / scale_m), -127, 127)
// (correctly rounded division, ties to even; a row of zeros has scale 0 and
// codes 0), and the per-group code sums S_mg = sum_{k in g} q_mk that fold
// the weights' zero point out of the integer dot products.
//
// Layout of the codes (what the W4A8 GEMV reads): int8 [M, K] row-major,
// with the channels of every 8-channel chunk stored in the order
// 0, 4, 1, 5, 2, 6, 3, 7 -- the order in which the two nibble masks of a
// packed weight word yield its codes (low nibbles: channels 0, 4, 1, 5;
// high nibbles: 2, 6, 3, 7), so a code word and an activation word pair up
// byte for byte in the tensor-core instruction.
#include "w4_common.cuh"
#include "w4_kernels.h"

namespace w4 {

namespace {

constexpr int kActThreads = 256;

__device__ __forceinline__ void bf16x8(const uint4 r, float (&v)[8]) {
  const uint32_t u[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(u[i] << 16);
    v[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
  }
}

// One CTA per token row.
__global__ void __launch_bounds__(kActThreads)
    quantize_act_int8_kernel(const __nv_bfloat16* __restrict__ x, int64_t K,
                             int8_t* __restrict__ xq, int32_t* __restrict__ xsum,
                             float* __restrict__ xscale) {
  __shared__ float red[kActThreads / 32];
  const int64_t m = blockIdx.x;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const uint4* xr = reinterpret_cast<const uint4*>(x + m * K);
  const int64_t chunks = K / 8;

  float a = 0.f;
  for (int64_t c = tid; c < chunks; c += kActThreads) {
    float v[8];
    bf16x8(__ldg(xr + c), v);
#pragma unroll
    for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(v[i]));
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  if (lane == 0) red[tid >> 5] = a;
  __syncthreads();
  float amax = red[0];
#pragma unroll
  for (int w = 1; w < kActThreads / 32; ++w) amax = fmaxf(amax, red[w]);
  const float scale = __fdiv_rn(amax, 127.0f);
  if (tid == 0) xscale[m] = scale;

  // Chunk c = base + tid: the 16 chunks of a group are 16 consecutive lanes
  // of one warp (K is a multiple of 128, so a group is whole or absent).
  const int64_t G = K / 128;
  uint2* qr = reinterpret_cast<uint2*>(xq + m * K);
  for (int64_t base = 0; base < chunks; base += kActThreads) {
    const int64_t c = base + tid;
    const bool valid = c < chunks;
    int q[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (valid && scale > 0.f) {
      float v[8];
      bf16x8(__ldg(xr + c), v);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        q[i] = min(127, max(-127, __float2int_rn(__fdiv_rn(v[i], scale))));
    }
    int s = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) s += q[i];
    if (valid) {
      // bytes in channel order 0, 4, 1, 5 | 2, 6, 3, 7
      const uint32_t lo = (q[0] & 0xFF) | ((q[4] & 0xFF) << 8) | ((q[1] & 0xFF) << 16) |
                          (static_cast<uint32_t>(q[5] & 0xFF) << 24);
      const uint32_t hi = (q[2] & 0xFF) | ((q[6] & 0xFF) << 8) | ((q[3] & 0xFF) << 16) |
                          (static_cast<uint32_t>(q[7] & 0xFF) << 24);
      qr[c] = make_uint2(lo, hi);
    }
#pragma unroll
    for (int o = 8; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (valid && (lane & 15) == 0) xsum[m * G + c / 16] = s;
  }
}

}  // namespace

cudaError_t launch_quantize_act_int8(const void* x, int64_t M, int64_t K, int8_t* xq,
                                     int32_t* xsum, float* xscale, cudaStream_t stream) {
  if (M < 1 || M > 0x7FFFFFFF) return cudaErrorInvalidValue;
  quantize_act_int8_kernel<<<static_cast<unsigned>(M), kActThreads, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(x), K, xq, xsum, xscale);
  return cudaGetLastError();
}

}  // namespace w4
