// Quantize + pack kernel: bf16 weight [N, K] -> int32 codes [N, K/8],
// fp16 scales [N, K/128], fp16 zeros [N, K/128] (asymmetric).
//
// HBM-bound: 2 bytes read and 0.5 + 4/128 (asymmetric) bytes written per
// weight.  A tensor is a flat sequence of N*K/128 contiguous 256-byte groups;
// a chunk is 32 consecutive groups (8 KB) and one lane owns one group of it.
// Each warp runs its own pipeline: lane 0 streams chunks into a ring of
// shared-memory stages with 1-D bulk copies (TMA engine, mbarrier
// completion), and the warp makes two passes over each stage, the group
// statistics and then the codes.  With a whole group per lane, the group
// parameters (two IEEE divisions and a reciprocal) are computed once per 128
// weights and no shuffles are needed.
//
// Lane l reads its 16-byte pieces in an order XOR-ed with l & 7, so the
// eight lanes of each shared-memory phase always hit eight different bank
// groups.
#include "quant_group.cuh"
#include "w4_kernels.h"

namespace w4 {

namespace {

#ifndef W4_QUANT_WARPS
#define W4_QUANT_WARPS 14
#endif
constexpr int kQWarps = W4_QUANT_WARPS;             // warps per CTA
constexpr int kQThreads = 32 * kQWarps;
#ifndef W4_QUANT_CTAS
#define W4_QUANT_CTAS 1
#endif
#ifndef W4_QUANT_STAGES
#define W4_QUANT_STAGES 2
#endif
constexpr int kQCtasPerSm = W4_QUANT_CTAS;
constexpr int kQStages = W4_QUANT_STAGES;           // ring depth per warp
constexpr int kChunkGroups = 32;                    // one group per lane
constexpr int kChunkBytes = kChunkGroups * 256;     // 8 KB of bf16
constexpr int kRingBytes = kQWarps * kQStages * kChunkBytes;
constexpr int kQSmemBytes = kRingBytes + kQWarps * kQStages * 8 + kQWarps * 4;
constexpr unsigned kKernelIdQuantize = 4;

// 1-D bulk copy global -> this CTA's shared memory, completing on `bar`.
// Both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(dst), "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 r;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "r"(addr));
  return r;
}

__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  float2 r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;"
      : "=l"(*reinterpret_cast<unsigned long long*>(&r))
      : "l"(*reinterpret_cast<unsigned long long*>(&a)),
        "l"(*reinterpret_cast<unsigned long long*>(&b)),
        "l"(*reinterpret_cast<unsigned long long*>(&c)));
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
__device__ __forceinline__ uint32_t clamp_codes_s16x2(uint32_t p) {
  uint32_t r;
  asm("max.s16x2 %0, %1, %2;" : "=r"(r) : "r"(p), "r"(0u));
  asm("min.s16x2 %0, %1, %2;" : "=r"(r) : "r"(r), "r"(0x000F000Fu));
  return r;
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

// The eight values of one 16-byte piece as four channel pairs, times the AWQ
// scale when there is one (binary32 products, as the definition has them).
template <bool HAS_S>
__device__ __forceinline__ void piece_values(const uint4 r, const float* s8, float2 (&v)[4]) {
  const uint32_t u[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
  for (int p = 0; p < 4; ++p)
    v[p] = make_float2(__uint_as_float(u[p] << 16), __uint_as_float(u[p] & 0xFFFF0000u));
  if (HAS_S) {
    const float4 s0 = __ldg(reinterpret_cast<const float4*>(s8));
    const float4 s1 = __ldg(reinterpret_cast<const float4*>(s8) + 1);
    v[0] = mul2(v[0], make_float2(s0.x, s0.y));
    v[1] = mul2(v[1], make_float2(s0.z, s0.w));
    v[2] = mul2(v[2], make_float2(s1.x, s1.y));
    v[3] = mul2(v[3], make_float2(s1.z, s1.w));
  }
}

// The word of eight codes of one piece through the exact per-value path.
// Everything is passed by value so the (rare) call needs no stack copy of
// the caller's values.
template <bool HAS_S>
__device__ __noinline__ uint32_t exact_word(const uint4 r, const float* s8, const GroupQ g) {
  float2 v[4];
  piece_values<HAS_S>(r, s8, v);
  uint32_t w = 0u;
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const uint32_t c0 = code_of(v[p].x, g), c1 = code_of(v[p].y, g);
    w |= (c0 | (c1 << 16)) << (4 * p);
  }
  return w;
}

// Stores the sixteen words of a group, held in read order: word i is piece
// ci = i ^ rot, which sits at position (i & 3) ^ (rot & 3) of 16-byte block
// (i >> 2) ^ (rot >> 2); two conditional swaps put each block in order.
__device__ __forceinline__ void store_words(const uint32_t (&wd)[16], int rot, uint4* qrow,
                                            bool valid) {
#pragma unroll
  for (int blk = 0; blk < 4; ++blk) {
    uint32_t w4[4] = {wd[4 * blk], wd[4 * blk + 1], wd[4 * blk + 2], wd[4 * blk + 3]};
    if (rot & 1) {
      uint32_t t = w4[0]; w4[0] = w4[1]; w4[1] = t;
      t = w4[2]; w4[2] = w4[3]; w4[3] = t;
    }
    if (rot & 2) {
      uint32_t t = w4[0]; w4[0] = w4[2]; w4[2] = t;
      t = w4[1]; w4[1] = w4[3]; w4[3] = t;
    }
    if (valid) qrow[blk ^ (rot >> 2)] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
  }
}

// The code of one value through the exact per-value path (quant_group.cuh),
// out of line: only values within about 2^-18 relative of a half-integer
// quotient that do not sit exactly on it come here.
__device__ __noinline__ uint32_t code_exact(float x, const GroupQ g) { return code_of(x, g); }

// Recomputes the word of one piece whose two bracketing roundings disagreed
// for at least one value.  Where they disagree, a half-integer T lies between
// v*rcp_lo and v*rcp_hi (the fma results differ by exactly one, so
// T = min - Mz + 1/2).  Most such values sit exactly on it: bf16 values times
// fp16 scales hit half-integer quotients about once in 1300 values.
// v = T * scale exactly iff fma(-T, scale, v) is zero (the exact difference of
// two multiples of 2^-150 cannot round to zero otherwise); then fl(q) = q = T
// and rint(T) (ties to even) is the code before the zero point.  Any other
// value takes the exact per-value path.
template <bool HAS_S>
__device__ __forceinline__ uint32_t repair_word(const uint4 r, const float* s8, const GroupQ& g,
                                                float rh, float rl, float mz) {
  const uint32_t u[4] = {r.x, r.y, r.z, r.w};
  uint32_t word = 0u;
#pragma unroll
  for (int b = 0; b < 8; ++b) {  // channel b of the piece
    float x = __uint_as_float((b & 1) ? (u[b >> 1] & 0xFFFF0000u) : (u[b >> 1] << 16));
    if (HAS_S) x = __fmul_rn(x, __ldg(s8 + b));
    const float a = __fmaf_rn(x, rh, mz), z = __fmaf_rn(x, rl, mz);
    uint32_t code;
    if (a == z) {
      const float q = __fsub_rn(a, 12582912.0f);  // rint(x / scale) + zero, exact
      code = q >= 15.0f ? 15u : (q > 0.0f ? static_cast<uint32_t>(q) : 0u);
    } else {
      const float t = __fadd_rn(__fsub_rn(fminf(a, z), mz), 0.5f);  // exact
      if (__fmaf_rn(-t, g.sc, x) == 0.0f) {
        const float q = __fadd_rn(rintf(t), g.zero);
        code = q >= 15.0f ? 15u : (q > 0.0f ? static_cast<uint32_t>(q) : 0u);
      } else {
        code = code_exact(x, g);
      }
    }
    word |= code << (4 * (b >> 1) + 16 * (b & 1));  // nibble of channel b
  }
  return word;
}

// Pass 2 of one group: its sixteen code words.  Piece i of the group
// (16 bytes, 8 values, one word) is read in the order ci = i ^ rot, at
// pm[i & 7] + 128 * (i >> 3) with pm[m] = group + 16 (m ^ rot).  The fast
// path runs on every piece and marks the pieces whose bracketing roundings
// disagree; a repair loop then redoes one marked word per lane per round, so
// the warp takes as many rounds as its busiest lane needs (about one per
// chunk).  Word ci sits at position (i & 3) ^ (rot & 3) of 16-byte block
// (i >> 2) ^ (rot >> 2); two conditional swaps put each block in order.
template <bool HAS_S>
__device__ __forceinline__ void code_pass(const uint32_t (&pm)[8], uint32_t gsrc, int rot,
                                          const float* s_grp, float rh, float rl, float mz,
                                          bool big, const GroupQ& g, uint4* qrow, bool valid) {
  const float2 rh2 = make_float2(rh, rh), rl2 = make_float2(rl, rl), mz2 = make_float2(mz, mz);
  uint32_t wd[16];
  uint32_t marks = big ? 0xFFFFu : 0u;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float2 v[4];
    piece_values<HAS_S>(lds128(pm[i & 7] + 128 * (i >> 3)),
                        HAS_S ? s_grp + 8 * (i ^ rot) : nullptr, v);
    uint32_t word = 0u, diff = 0u;
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const float2 a = fma2(v[p], rh2, mz2);
      const float2 z = fma2(v[p], rl2, mz2);
      const uint32_t pa = __byte_perm(__float_as_uint(a.x), __float_as_uint(a.y), 0x5410);
      const uint32_t pz = __byte_perm(__float_as_uint(z.x), __float_as_uint(z.y), 0x5410);
      diff |= pa ^ pz;
      word += clamp_codes_s16x2(pa) << (4 * p);  // disjoint nibbles
    }
    wd[i] = word;
    marks |= (diff != 0u ? 1u : 0u) << i;
  }
  while (__any_sync(0xffffffffu, marks != 0u)) {
    if (marks != 0u) {
      const int i = __ffs(marks) - 1;
      marks &= marks - 1u;
      const int ci = i ^ rot;
      const uint4 r = lds128(gsrc + 16 * ci);
      const float* s8 = HAS_S ? s_grp + 8 * ci : nullptr;
      const uint32_t w = big ? exact_word<HAS_S>(r, s8, g) : repair_word<HAS_S>(r, s8, g, rh, rl, mz);
#pragma unroll
      for (int q = 0; q < 16; ++q) wd[q] = (q == i) ? w : wd[q];
    }
  }
  store_words(wd, rot, qrow, valid);
}

// Pass 2 for bf16 values (no AWQ scale): the correctly rounded binary32
// quotient without a division.  With rcp = fl(1/scale), q0 = fl(v * rcp),
// r = v - q0 * scale (exact, one fma) and q1 = fl(q0 + r * rcp) (one fma),
// q1 equals fl(v / scale) for every bf16 v and fp16 scale: the correction
// step of P. Markstein ("Computation of elementary functions on the IBM RISC
// System/6000 processor", 1990), checked here exhaustively with exact
// rational arithmetic over all 2^7 x 2^10 significand pairs (the result is
// invariant under power-of-two scaling of either operand away from
// underflow; where v is so small that q underflows, |q| is far below 1/2 and
// every candidate code is the zero point).  fl(q1 + 1.5 * 2^23) then rounds q1
// to an integer, ties to even, as rint does, and adding the zero point to
// that integer-valued sum is exact; its low 16 bits are the code before the
// clamp.  Groups with |v * rcp| >= 2^14 go through the exact per-value path.
__device__ __forceinline__ void code_pass_bf16(const uint32_t (&pm)[8], uint32_t gsrc, int rot,
                                               bool big, const GroupQ& g, uint4* qrow,
                                               bool valid) {
  const float2 rcp2 = make_float2(g.rcp, g.rcp), nsc2 = make_float2(-g.sc, -g.sc);
  const float2 m2 = make_float2(12582912.0f, 12582912.0f), z2 = make_float2(g.zero, g.zero);
  uint32_t wd[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float2 v[4];
    piece_values<false>(lds128(pm[i & 7] + 128 * (i >> 3)), nullptr, v);
    uint32_t word = 0u;
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const float2 q0 = mul2(v[p], rcp2);
      const float2 r = fma2(q0, nsc2, v[p]);
      const float2 q1 = fma2(r, rcp2, q0);
      const float2 c = add2(add2(q1, m2), z2);
      const uint32_t pc = __byte_perm(__float_as_uint(c.x), __float_as_uint(c.y), 0x5410);
      word += clamp_codes_s16x2(pc) << (4 * p);  // disjoint nibbles
    }
    wd[i] = word;
  }
  if (big) {
#pragma unroll 1
    for (int i = 0; i < 16; ++i) {
      const uint32_t w = exact_word<false>(lds128(gsrc + 16 * (i ^ rot)), nullptr, g);
#pragma unroll
      for (int q = 0; q < 16; ++q) wd[q] = (q == i) ? w : wd[q];
    }
  }
  store_words(wd, rot, qrow, valid);
}

// Codes, fast path.  rcp = fl(1/scale) is within 2^-24 relative of 1/scale;
// rcp_hi = fl(rcp (1 + 2^-18)) and rcp_lo = fl(rcp (1 - 2^-18)) then differ
// from it by more than 2^-19 relative, so for every value the exact quotient
// q = v/scale and its binary32 rounding fl(q) lie strictly between v*rcp_lo
// and v*rcp_hi.  With Mz = 1.5*2^23 + zero, fma(v, rcp_x, Mz) rounds the exact
// product plus Mz to an integer, whose low 16 bits are that integer minus
// 1.5*2^23 as a signed 16-bit number (|v * rcp| < 2^14 is checked per group).
// Rounding is monotone, so when both ends give the same integer no
// half-integer lies between them, and it equals rint(fl(q)) + zero.  Where
// the two ends differ (a few values in 10^5), the word of eight codes is
// recomputed on the exact path of quant_group.cuh.  Two codes share a
// register (pair of adjacent channels 2p, 2p+1), are clamped to 0..15 with
// packed 16-bit min/max, and in the canonical nibble order land in nibbles
// (p, p+4) of the word: one shift by 4p.
template <bool SYM, bool HAS_S>
__global__ void __launch_bounds__(kQThreads, kQCtasPerSm)
    quantize_pack_kernel(const __grid_constant__ QuantBatch b, unsigned* err) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  const int rot = lane & 7;
  const uint32_t ring = smem_u32(smem) + wib * kQStages * kChunkBytes;
  const uint32_t bar0 = smem_u32(smem + kRingBytes) + wib * kQStages * 8;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kRingBytes +
                                                             kQWarps * kQStages * 8) + wib;
  const int64_t warp = static_cast<int64_t>(blockIdx.x) * kQWarps + wib;
  const int64_t n_warps = static_cast<int64_t>(gridDim.x) * kQWarps;
  const int64_t n_chunks = b.unit_start[b.count];

  if (lane == 0) {
#pragma unroll
    for (int s = 0; s < kQStages; ++s) mbar_init(bar0 + 8 * s, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncwarp();

  // Chunk c -> its tensor.  A warp's chunks only increase, so each cursor
  // moves forward through the tensors.
  auto advance = [&](int& it, int64_t c) {
    while (it + 1 < b.count && b.unit_start[it + 1] <= c) ++it;
  };
  int it_load = 0;
  int64_t issued = 0;  // chunks this warp has requested (lane 0's count)
  auto issue = [&](int64_t c) {
    advance(it_load, c);
    const int64_t g0 = kChunkGroups * (c - b.unit_start[it_load]);
    const int64_t left = b.n_groups[it_load] - g0;
    const uint32_t bytes = static_cast<uint32_t>(left < kChunkGroups ? left : kChunkGroups) * 256u;
    const int s = static_cast<int>(issued % kQStages);
    mbar_arrive_expect_tx(bar0 + 8 * s, bytes);
    bulk_load(ring + s * kChunkBytes, static_cast<const uint8_t*>(b.w[it_load]) + g0 * 256, bytes,
              bar0 + 8 * s);
    ++issued;
  };
  if (lane == 0) {
    for (int j = 0; j < kQStages; ++j)
      if (warp + j * n_warps < n_chunks) issue(warp + j * n_warps);
  }

  int it = 0;
  int64_t k = 0;  // chunks consumed
  for (int64_t c = warp; c < n_chunks; c += n_warps, ++k) {
    const int s = static_cast<int>(k % kQStages);
    const bool ok = mbar_wait(bar0 + 8 * s, static_cast<uint32_t>(k / kQStages) & 1u, abort_flag,
                              err, kKernelIdQuantize);
    // A lane that gave up sets the warp's abort flag, which ends every other
    // lane's wait too; the whole warp leaves together.
    if (!__all_sync(0xffffffffu, ok)) break;
    advance(it, c);
    const int64_t gi = kChunkGroups * (c - b.unit_start[it]) + lane;
    const bool valid = gi < b.n_groups[it];
    const uint32_t gsrc = ring + s * kChunkBytes + lane * 256;
    uint32_t pm[8];  // pm[m] = address of piece m ^ rot; piece i is at pm[i & 7] + 128 (i >> 3)
#pragma unroll
    for (int m = 0; m < 8; ++m) pm[m] = gsrc + 16 * (m ^ rot);
    const float* s_grp = nullptr;
    if (HAS_S) {
      s_grp = b.s[it];
      if (s_grp != nullptr) s_grp += (valid ? gi % b.groups_per_row[it] : 0) * 128;
    }

    // Pass 1: group statistics.
    float gmax, gmin = 0.f;
    if (!HAS_S || s_grp == nullptr) {
      // On the raw bf16 pairs (exact: max/min only compare), four
      // independent accumulators, one per register of a piece.
      uint32_t mx[4], mn[4];
      {
        const uint4 r = lds128(pm[0]);
        const uint32_t u[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          mx[q] = SYM ? (u[q] & 0x7FFF7FFFu) : u[q];
          mn[q] = u[q];
        }
      }
#pragma unroll
      for (int i = 1; i < 16; ++i) {
        const uint4 r = lds128(pm[i & 7] + 128 * (i >> 3));
        const uint32_t u[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          mx[q] = bmax2(mx[q], SYM ? (u[q] & 0x7FFF7FFFu) : u[q]);
          if (!SYM) mn[q] = bmin2(mn[q], u[q]);
        }
      }
      const uint32_t bx = bmax2(bmax2(mx[0], mx[1]), bmax2(mx[2], mx[3]));
      gmax = fmaxf(__uint_as_float(bx << 16), __uint_as_float(bx & 0xFFFF0000u));
      if (!SYM) {
        const uint32_t bn = bmin2(bmin2(mn[0], mn[1]), bmin2(mn[2], mn[3]));
        gmin = fminf(__uint_as_float(bn << 16), __uint_as_float(bn & 0xFFFF0000u));
      }
    } else {
      float mx = -INFINITY, mn = INFINITY, ax = 0.f;
#pragma unroll 4
      for (int i = 0; i < 16; ++i) {
        const int ci = i ^ rot;
        float2 v[4];
        piece_values<HAS_S>(lds128(pm[i & 7] + 128 * (i >> 3)), s_grp + 8 * ci, v);
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          if (SYM) {
            ax = fmaxf(ax, fmaxf(fabsf(v[p].x), fabsf(v[p].y)));
          } else {
            mx = fmaxf(mx, fmaxf(v[p].x, v[p].y));
            mn = fminf(mn, fminf(v[p].x, v[p].y));
          }
        }
      }
      gmax = SYM ? ax : mx;
      gmin = mn;
    }
    const float* srow = b.shrink_rows[it];
    // (lanes past the last group read no row ratio)
    const float shrink =
        (srow && valid) ? __ldg(srow + gi / b.groups_per_row[it]) : b.shrink[it];
    const GroupQ g = group_params<SYM>(gmax, gmin, shrink);
    const float amax = SYM ? gmax : fmaxf(fabsf(gmax), fabsf(gmin));
    const bool big = !(__fmul_rn(amax, g.rcp) < 16384.0f);
    const float rh = __fmul_rn(g.rcp, 1.000003814697265625f);  // 1 + 2^-18
    const float rl = __fmul_rn(g.rcp, 0.999996185302734375f);  // 1 - 2^-18
    const float mz = 12582912.0f + g.zero;                     // exact

    // Pass 2: codes.
    uint4* qrow = static_cast<uint4*>(b.qw[it]) + gi * 4;
    if (HAS_S && s_grp != nullptr)
      code_pass<true>(pm, gsrc, rot, s_grp, rh, rl, mz, big, g, qrow, valid);
    else
      code_pass_bf16(pm, gsrc, rot, big, g, qrow, valid);
    if (valid) {
      b.scales[it][gi] = g.s16;
      if (!SYM) b.zeros[it][gi] = g.z16;
    }
    // Every lane is done with this stage: refill it.
    __syncwarp();
    if (lane == 0 && c + kQStages * n_warps < n_chunks) issue(c + kQStages * n_warps);
  }
  // After a timeout: wait (bounded) for this warp's copies still in flight
  // before the CTA's shared memory goes away.
  if (lane == 0 && *abort_flag) {
    int dummy = 0;
    for (int64_t q = k; q < issued; ++q)
      mbar_wait(bar0 + 8 * static_cast<int>(q % kQStages),
                static_cast<uint32_t>(q / kQStages) & 1u, &dummy, err, kKernelIdQuantize,
                kWaitLimitNs / 4);
  }
}

template <bool SYM, bool HAS_S>
cudaError_t launch_t(const QuantBatch& b, cudaStream_t stream, int num_sms, unsigned* err) {
  auto kern = quantize_pack_kernel<SYM, HAS_S>;
  static bool attr_done[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!attr_done[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kQSmemBytes);
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  const int64_t n_chunks = b.unit_start[b.count];
  int64_t blocks = (n_chunks + kQWarps - 1) / kQWarps;
  // Persistent grid: every CTA resident at once, each warp striding over
  // the chunks with its ring of copies running ahead.
  const int64_t cap = static_cast<int64_t>(num_sms) * kQCtasPerSm;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  kern<<<static_cast<unsigned>(blocks), kQThreads, kQSmemBytes, stream>>>(b, err);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_quantize_pack_batch(const QuantBatch& b, bool symmetric, cudaStream_t stream,
                                       int num_sms, unsigned* err) {
  bool any_s = false;
  for (int i = 0; i < b.count; ++i) any_s = any_s || b.s[i] != nullptr;
  if (symmetric)
    return any_s ? launch_t<true, true>(b, stream, num_sms, err)
                 : launch_t<true, false>(b, stream, num_sms, err);
  return any_s ? launch_t<false, true>(b, stream, num_sms, err)
               : launch_t<false, false>(b, stream, num_sms, err);
}

void quant_batch_add(QuantBatch& b, const void* w, int64_t N, int64_t K, const float* s,
                     float shrink, int32_t* qweight, uint16_t* scales, uint16_t* zeros,
                     const float* shrink_rows) {
  const int i = b.count;
  b.w[i] = w;
  b.s[i] = s;
  b.shrink[i] = shrink;
  b.shrink_rows[i] = shrink_rows;
  b.qw[i] = qweight;
  b.scales[i] = scales;
  b.zeros[i] = zeros;
  b.n_groups[i] = N * (K / 128);
  b.groups_per_row[i] = K / 128;
  b.unit_start[i + 1] = b.unit_start[i] + (b.n_groups[i] + kChunkGroups - 1) / kChunkGroups;
  b.count = i + 1;
}

}  // namespace w4
