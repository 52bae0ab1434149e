// Per-group int4 RTN quantization math, shared by the quantize+pack kernel
// and the AWQ candidate builder.  A group is 128 consecutive input channels
// of one output row, held by 16 lanes (8 values each) of a warp.
//
// Definition ("ghostchoir/rebuttal_w4g128_awq_w2" model card, 'Model Details'
// row 'Scheme': weight-only 4-bit, group 128, asymmetric zero point;
// "GotoAI-Inc/Qwen3.6-27B-W4A16" model card, opening paragraph: symmetric
// int4 g128), all in IEEE binary32, round to nearest even, no contraction:
//   asymmetric: scale = fp16(max(r*max - r*min, 1e-5) / 15)
//               zero  = clamp(rint(-(r*min) / scale), 0, 15)
//   symmetric:  scale = fp16(max(r*absmax, 1e-5) / 7),  zero = 8
//   code = clamp(rint(v / scale) + zero, 0, 15),  scale = stored fp16 value.
#pragma once

#include "w4_common.cuh"

namespace w4 {

struct GroupQ {
  float sc;      // stored scale widened to fp32
  float rcp;     // fl(1 / sc)
  float zero;    // integer-valued zero point
  uint16_t s16;  // fp16 bits of the scale
  uint16_t z16;  // fp16 bits of the zero (asymmetric)
};

// Reduction over the 16 lanes of a half warp (xor offsets stay inside it).
__device__ __forceinline__ float hw_max(float a) {
#pragma unroll
  for (int o = 8; o; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  return a;
}
__device__ __forceinline__ float hw_min(float a) {
#pragma unroll
  for (int o = 8; o; o >>= 1) a = fminf(a, __shfl_xor_sync(0xffffffffu, a, o));
  return a;
}

// Group parameters from the group's (unshrunk) max and min (asymmetric) or
// absmax (symmetric; pass it as gmax).
template <bool SYM>
__device__ __forceinline__ GroupQ group_params(float gmax, float gmin, float shrink) {
  GroupQ g;
  float scale32;
  float mn = 0.f;
  if (SYM) {
    const float a = __fmul_rn(shrink, gmax);
    scale32 = __fdiv_rn(fmaxf(a, 1e-5f), 7.0f);
  } else {
    const float mx = __fmul_rn(shrink, gmax);
    mn = __fmul_rn(shrink, gmin);
    scale32 = __fdiv_rn(fmaxf(__fsub_rn(mx, mn), 1e-5f), 15.0f);
  }
  const __half h = __float2half_rn(scale32);
  g.s16 = __half_as_ushort(h);
  g.sc = __half2float(h);
  g.rcp = __frcp_rn(g.sc);
  if (SYM) {
    g.zero = 8.0f;
    g.z16 = 0x4800;  // fp16 8.0
  } else {
    const float zr = rintf(__fdiv_rn(-mn, g.sc));
    const int zi = zr >= 15.0f ? 15 : (zr > 0.0f ? static_cast<int>(zr) : 0);  // NaN -> 0
    g.zero = static_cast<float>(zi);
    g.z16 = __half_as_ushort(__float2half_rn(static_cast<float>(zi)));
  }
  return g;
}

// rint(fl(v / sc)) without a division on the common path.
//
// t = fl(v * fl(1/sc)) is within 1.5 * 2^-23 * |v/sc| (plus nothing) of the
// exact quotient y, and fl(y) within 2^-24 * |y|.  If t is more than
// 2^-21 * |t| away from every half-integer tie, then t, y and fl(y) all lie
// strictly inside the same interval between consecutive ties, so
// rint(fl(y)) == rint(t).  Otherwise (about one value in 10^5, and every
// value of a degenerate group whose quotients exceed 2^20) the correctly
// rounded division decides.  0.5 - |t - rint(t)| is computed exactly for
// |t| >= 1/4 and is above the threshold for |t| < 1/4.
__device__ __forceinline__ float rint_quotient(float v, float sc, float rcp) {
  const float t = __fmul_rn(v, rcp);
  float rt = rintf(t);
  const float dtie = __fsub_rn(0.5f, fabsf(__fsub_rn(t, rt)));
  if (!(dtie > __fmul_rn(fabsf(t), 4.76837158203125e-07f))) {  // 2^-21
    rt = rintf(__fdiv_rn(v, sc));
  }
  return rt;
}

// Code of one value: clamp(rint(v/sc) + zero, 0, 15).
__device__ __forceinline__ uint32_t code_of(float v, const GroupQ& g) {
  const float q = __fadd_rn(rint_quotient(v, g.sc, g.rcp), g.zero);
  return q >= 15.0f ? 15u : (q > 0.0f ? static_cast<uint32_t>(q) : 0u);  // NaN -> 0
}

// Canonical nibble position of channel offset j (0..7) inside its int32
// word: nibbles low->high hold channel offsets 0,2,4,6,1,3,5,7.
__host__ __device__ constexpr int nibble_pos(int j) { return (j >> 1) + 4 * (j & 1); }

// Widens 8 bf16 (one uint4) to fp32.
__device__ __forceinline__ void bf16x8_to_f32(const uint4 r, float (&v)[8]) {
  const uint32_t u[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[2 * i] = __uint_as_float(u[i] << 16);
    v[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
  }
}

}  // namespace w4
