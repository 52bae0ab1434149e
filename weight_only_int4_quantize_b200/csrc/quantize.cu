// Quantize + pack kernel: bf16 weight [N, K] -> int32 codes [N, K/8],
// fp16 scales [N, K/128], fp16 zeros [N, K/128] (asymmetric).
//
// HBM-bound: 2 bytes read and 0.5 + 4/128 (asymmetric) bytes written per
// weight.  The weight is a sequence of N*K/128 contiguous 256-byte groups;
// a lane quad owns one group per step, each lane 64 contiguous bytes (32
// values), so a warp reads 2 KB of consecutive memory and the 16 packed
// words of a group are four contiguous 16-byte stores.  Group min/max use
// quad shuffles (on packed bf16 pairs when no AWQ scale is applied).
#include "quant_group.cuh"
#include "w4_kernels.h"

namespace w4 {

namespace {

constexpr int kQuantThreads = 256;

__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  float2 r;
  asm("mul.rn.f32x2 %0, %1, %2;"
      : "=l"(*reinterpret_cast<unsigned long long*>(&r))
      : "l"(*reinterpret_cast<unsigned long long*>(&a)),
        "l"(*reinterpret_cast<unsigned long long*>(&b)));
  return r;
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  float2 r;
  asm("add.rn.f32x2 %0, %1, %2;"
      : "=l"(*reinterpret_cast<unsigned long long*>(&r))
      : "l"(*reinterpret_cast<unsigned long long*>(&a)),
        "l"(*reinterpret_cast<unsigned long long*>(&b)));
  return r;
}
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  float2 r;
  asm("sub.rn.f32x2 %0, %1, %2;"
      : "=l"(*reinterpret_cast<unsigned long long*>(&r))
      : "l"(*reinterpret_cast<unsigned long long*>(&a)),
        "l"(*reinterpret_cast<unsigned long long*>(&b)));
  return r;
}
__device__ __forceinline__ uint32_t clamp_codes_s16x2(uint32_t p) {
  uint32_t r;
  asm("max.s16x2 %0, %1, %2;" : "=r"(r) : "r"(p), "r"(0u));
  asm("min.s16x2 %0, %1, %2;" : "=r"(r) : "r"(r), "r"(0x000F000Fu));
  return r;
}

// Reduction over the 4 lanes of a lane quad.
__device__ __forceinline__ float quad_max(float a) {
  a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
  return fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
}
__device__ __forceinline__ float quad_min(float a) {
  a = fminf(a, __shfl_xor_sync(0xffffffffu, a, 2));
  return fminf(a, __shfl_xor_sync(0xffffffffu, a, 1));
}
__device__ __forceinline__ uint32_t bmax2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t bmin2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("min.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

// One group = 128 contiguous values held by a lane quad, 32 per lane
// (channels 32*l4 .. 32*l4+31 of the group, in adjacent pairs).  A warp
// quantizes eight consecutive groups per iteration.
//
// Codes, fast path: with t = v * fl(1/scale) and Mz = 1.5*2^23 + zero,
// fl(t + Mz) = Mz + rint(t) whenever t is not within 2^-16 of a half-integer
// tie (so the tie-breaking parity of Mz never matters), and its low 16 bits
// are rint(t) + zero as a signed 16-bit integer (|t| < 2^14 is checked per
// group).  Two such codes are packed into one register, clamped to 0..15 with
// packed 16-bit min/max, and in the canonical nibble order the pair of
// adjacent channels (2i, 2i+1) belongs in nibbles (i, i+4): one shift by 4i.
// t lies within 1.5 * 2^-23 * |v/scale| of the exact quotient, so for
// |t| < 17 a distance above 2^-16 from every tie guarantees
// rint(fl(v/scale)) == rint(t); for |t| >= 17 the clamp saturates either way.
// Any lane with a value closer to a tie sends the whole warp through the
// exact path (correctly rounded division, as in quant_group.cuh).
template <bool SYM, bool HAS_S>
__global__ void __launch_bounds__(kQuantThreads, 3)
    quantize_pack_kernel(const __grid_constant__ QuantBatch b) {
  const int lane = threadIdx.x & 31;
  const int sub = lane >> 2;  // group of this quad within the warp's eight
  const int l4 = lane & 3;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kQuantThreads + threadIdx.x) >> 5;
  const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * kQuantThreads) >> 5;
  const int64_t n_units = b.unit_start[b.count];
  const float thr = 0.5f - 1.52587890625e-05f;  // 0.5 - 2^-16

  // Unit u (8 consecutive groups of one tensor) -> its tensor.
  auto item_of = [&](int64_t u) {
    int lo = 0, hi = b.count - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (b.unit_start[mid] <= u) lo = mid; else hi = mid - 1;
    }
    return lo;
  };
  // Software pipeline: the next unit's 64 bytes per lane are in flight while
  // the current unit is quantized.
  auto load_unit = [&](int64_t u, uint32_t (&dst)[16]) {
    uint4 r[4] = {};
    if (u < n_units) {
      const int it = item_of(u);
      const int64_t gi = 8 * (u - b.unit_start[it]) + sub;
      if (gi < b.n_groups[it]) {
        const uint4* src = static_cast<const uint4*>(b.w[it]) + gi * 16 + l4 * 4;
#pragma unroll
        for (int q = 0; q < 4; ++q) r[q] = ld_stream(src + q);
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      dst[4 * q] = r[q].x; dst[4 * q + 1] = r[q].y; dst[4 * q + 2] = r[q].z; dst[4 * q + 3] = r[q].w;
    }
  };
  uint32_t nxt[16];
  load_unit(warp, nxt);
  for (int64_t u = warp; u < n_units; u += n_warps) {
    const int it = item_of(u);
    const int64_t n_groups = b.n_groups[it];
    const int64_t gi = 8 * (u - b.unit_start[it]) + sub;
    const bool valid = gi < n_groups;
    const float shrink = b.shrink[it];
    const float* s = b.s[it];
    uint4* qw = static_cast<uint4*>(b.qw[it]);
    uint16_t* scales = b.scales[it];
    uint16_t* zeros = b.zeros[it];
    uint32_t raw[16];
#pragma unroll
    for (int p = 0; p < 16; ++p) raw[p] = nxt[p];
    load_unit(u + n_warps, nxt);
    float2 v[16];
#pragma unroll
    for (int p = 0; p < 16; ++p)
      v[p] = make_float2(__uint_as_float(raw[p] << 16), __uint_as_float(raw[p] & 0xFFFF0000u));
    GroupQ g;
    float amax;
    if (HAS_S) {
      if (s != nullptr) {
        const int64_t k0 = (gi % b.groups_per_row[it]) * 128 + l4 * 32;
        const float4* sp = reinterpret_cast<const float4*>(s + (valid ? k0 : 0));
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float4 sv = __ldg(sp + q);
          v[2 * q] = mul2(v[2 * q], make_float2(sv.x, sv.y));
          v[2 * q + 1] = mul2(v[2 * q + 1], make_float2(sv.z, sv.w));
        }
      }
      if (SYM) {
        float a = 0.f;
#pragma unroll
        for (int p = 0; p < 16; ++p) a = fmaxf(a, fmaxf(fabsf(v[p].x), fabsf(v[p].y)));
        amax = quad_max(a);
        g = group_params<true>(amax, 0.f, shrink);
      } else {
        float mx = v[0].x, mn = v[0].x;
#pragma unroll
        for (int p = 0; p < 16; ++p) {
          mx = fmaxf(mx, fmaxf(v[p].x, v[p].y));
          mn = fminf(mn, fminf(v[p].x, v[p].y));
        }
        mx = quad_max(mx);
        mn = quad_min(mn);
        g = group_params<false>(mx, mn, shrink);
        amax = fmaxf(fabsf(mx), fabsf(mn));
      }
    } else {
      // Group statistics on the raw bf16 pairs (exact: max/min only compare).
      uint32_t bx = raw[0], bn = raw[0];
      if (SYM) {
#pragma unroll
        for (int p = 0; p < 16; ++p) bx = bmax2(bx, raw[p] & 0x7FFF7FFFu);
      } else {
#pragma unroll
        for (int p = 1; p < 16; ++p) {
          bx = bmax2(bx, raw[p]);
          bn = bmin2(bn, raw[p]);
        }
      }
      const float mx = quad_max(fmaxf(__uint_as_float(bx << 16), __uint_as_float(bx & 0xFFFF0000u)));
      if (SYM) {
        amax = mx;
        g = group_params<true>(amax, 0.f, shrink);
      } else {
        const float mn =
            quad_min(fminf(__uint_as_float(bn << 16), __uint_as_float(bn & 0xFFFF0000u)));
        g = group_params<false>(mx, mn, shrink);
        amax = fmaxf(fabsf(mx), fabsf(mn));
      }
    }
    // Fast path.
    const float mz = 12582912.0f + g.zero;  // exact
    const float2 rcp2 = make_float2(g.rcp, g.rcp);
    const float2 mz2 = make_float2(mz, mz);
    float dmax = 0.f;
    uint32_t word[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int p = 0; p < 16; ++p) {
      const float2 t = mul2(v[p], rcp2);
      const float2 r = add2(t, mz2);
      const float2 d = sub2(t, sub2(r, mz2));
      dmax = fmaxf(dmax, fmaxf(fabsf(d.x), fabsf(d.y)));
      const uint32_t pair = __byte_perm(__float_as_uint(r.x), __float_as_uint(r.y), 0x5410);
      word[p >> 2] += clamp_codes_s16x2(pair) << (4 * (p & 3));
    }
    const bool bad = !(dmax < thr) || !(__fmul_rn(amax, g.rcp) < 16384.0f);
    if (__any_sync(0xffffffffu, bad)) {
      // Exact path for the whole warp (rare).
#pragma unroll
      for (int p = 0; p < 16; ++p) {
        if ((p & 3) == 0) word[p >> 2] = 0u;
        const uint32_t c0 = code_of(v[p].x, g), c1 = code_of(v[p].y, g);
        word[p >> 2] |= (c0 | (c1 << 16)) << (4 * (p & 3));
      }
    }
    // Scales / zeros of the eight groups: gathered into lanes 0 and 16.
    const uint32_t sz = static_cast<uint32_t>(g.s16) | (static_cast<uint32_t>(g.z16) << 16);
    const uint32_t sz1 = __shfl_down_sync(0xffffffffu, sz, 4);
    const uint32_t sz2 = __shfl_down_sync(0xffffffffu, sz, 8);
    const uint32_t sz3 = __shfl_down_sync(0xffffffffu, sz, 12);
    if (valid) qw[gi * 4 + l4] = make_uint4(word[0], word[1], word[2], word[3]);
    if ((lane & 15) == 0) {
      const int64_t g0 = gi;  // first of four consecutive groups
      if (g0 + 3 < n_groups) {
        *reinterpret_cast<uint2*>(scales + g0) =
            make_uint2((sz & 0xFFFFu) | (sz1 << 16), (sz2 & 0xFFFFu) | (sz3 << 16));
        if (!SYM)
          *reinterpret_cast<uint2*>(zeros + g0) =
              make_uint2((sz >> 16) | (sz1 & 0xFFFF0000u), (sz2 >> 16) | (sz3 & 0xFFFF0000u));
      } else {
        const uint32_t all[4] = {sz, sz1, sz2, sz3};
        for (int q = 0; q < 4 && g0 + q < n_groups; ++q) {
          scales[g0 + q] = static_cast<uint16_t>(all[q] & 0xFFFFu);
          if (!SYM) zeros[g0 + q] = static_cast<uint16_t>(all[q] >> 16);
        }
      }
    }
  }
}

}  // namespace

cudaError_t launch_quantize_pack_batch(const QuantBatch& b, bool symmetric, cudaStream_t stream,
                                       int num_sms) {
  const int64_t n_units = b.unit_start[b.count];
  int64_t blocks = (n_units + (kQuantThreads / 32) - 1) / (kQuantThreads / 32);
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;  // 8 x 256 threads per SM
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  bool any_s = false;
  for (int i = 0; i < b.count; ++i) any_s = any_s || b.s[i] != nullptr;
  dim3 grid(static_cast<unsigned>(blocks)), block(kQuantThreads);
  if (symmetric) {
    if (any_s) quantize_pack_kernel<true, true><<<grid, block, 0, stream>>>(b);
    else       quantize_pack_kernel<true, false><<<grid, block, 0, stream>>>(b);
  } else {
    if (any_s) quantize_pack_kernel<false, true><<<grid, block, 0, stream>>>(b);
    else       quantize_pack_kernel<false, false><<<grid, block, 0, stream>>>(b);
  }
  return cudaGetLastError();
}

void quant_batch_add(QuantBatch& b, const void* w, int64_t N, int64_t K, const float* s,
                     float shrink, int32_t* qweight, uint16_t* scales, uint16_t* zeros) {
  const int i = b.count;
  b.w[i] = w;
  b.s[i] = s;
  b.shrink[i] = shrink;
  b.qw[i] = qweight;
  b.scales[i] = scales;
  b.zeros[i] = zeros;
  b.n_groups[i] = N * (K / 128);
  b.groups_per_row[i] = K / 128;
  b.unit_start[i + 1] = b.unit_start[i] + (b.n_groups[i] + 7) / 8;
  b.count = i + 1;
}

}  // namespace w4
