// Decode W4A16 GEMV for up to 8 tokens, streaming from global memory:
// y[M, N] = x[M, K] . dequant(Wq)^T, HBM-bound on the packed weight stream
// (0.53125 B/weight asymmetric, 0.515625 symmetric).
//
// Work: a warp unit is 64 weight rows (four 16-row mma tiles) of one linear
// over one part of its K range.  Each linear's K is split into ks parts
// (ks in {1, 2, 4}, chosen per linear on the host so that units are of
// similar length); a bundle is the four warp units of one CTA step: four
// row blocks (ks = 1), two row blocks in two parts (ks = 2) or one row block
// in four parts.  The grid is persistent: CTA c takes bundles c, c + grid,
// ...; its warps run through them independently, and only the ks warps of
// one row block meet, at its end, to add their partial sums in shared
// memory in a fixed order (deterministic).
//
// A warp streams its units through its own ring of shared-memory slots,
// S groups ahead of use, with per-lane 16-byte asynchronous copies: each
// lane copies exactly the bytes of its own mma fragments (rows g and g + 8
// of each tile, channels 32t .. 32t+31 of the group) and one 4-byte word
// around each of its scale/zero values, and reads back only what it copied
// itself, so no barrier guards the ring.  The ring runs on across units, so
// a warp's memory stream does not stop between them and there is no per-CTA
// prologue.
//
// Per group a warp turns each tile into exact bf16 values 128 + q (one
// mask/OR per pair of codes), runs 8 mma.m16n8k16 against the x fragments
// (loaded from global memory one group ahead; x stays cached) and removes
// (128 + zero) * sum_k x_k, the sums coming from 8 mmas of all-ones rows
// shared by the four tiles:
//   sum_k (q - z) x_k = sum_k (128 + q) x_k - (128 + z) sum_k x_k.
// The scale multiplies the fp32 group result.  No global scratch; the only
// waits are the copy-group waits of a lane's own copies and the named
// barrier of the ks warps of a row block.
#include "w4_common.cuh"
#include "w4_kernels.h"

namespace w4 {

namespace {

constexpr int kStreamWarps = 4;
constexpr int kStreamThreads = 32 * kStreamWarps;
constexpr uint32_t kOnesBf16x2 = 0x3F803F80u;  // bf16x2 (1.0, 1.0)

// 16-byte asynchronous copy global -> shared (L2 only), zero-filled when
// `valid` is false (then no global memory is read; src is still a valid
// address of the same tensor).
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global.L2::256B [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
// 4-byte asynchronous copy global -> shared (cached in L1) of which the
// first `bytes` (0, 2 or 4) are read and the rest is zero-filled.
__device__ __forceinline__ void cp_async4_part(uint32_t dst, const void* src, uint32_t bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ uint32_t lds32s(uint32_t addr) {
  uint32_t r;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(r) : "r"(addr));
  return r;
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ uint4 lds128s(uint32_t addr) {
  uint4 r;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "r"(addr));
  return r;
}

__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                          uint32_t a3, uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One 16-row tile over one 128-channel group: 8 reduction steps.  Word j of
// each row (channels 8j .. 8j+7 of this lane's 32) feeds step 2j (code pairs
// at shifts 0 and 4) and step 2j+1 (shifts 8 and 12); the A fragment of a
// step is (w >> sh) & 0x000F000F | 0x43004300, bf16x2 (128 + q) pairs of
// adjacent channels (exact: bf16 has unit spacing on [128, 256)).
#define W4S_STEP(VA, VB, B0, B1, SH0, CIN)                                      \
  "shr.b32 s0, " VA ", " SH0 ";\n\t"                                            \
  "shr.b32 s1, " VB ", " SH0 ";\n\t"                                            \
  "shr.b32 s2, " VA ", " SH0 "+4;\n\t"                                          \
  "shr.b32 s3, " VB ", " SH0 "+4;\n\t"                                          \
  "lop3.b32 a0, s0, 0x000F000F, 0x43004300, 0xEA;\n\t"                          \
  "lop3.b32 a1, s1, 0x000F000F, 0x43004300, 0xEA;\n\t"                          \
  "lop3.b32 a2, s2, 0x000F000F, 0x43004300, 0xEA;\n\t"                          \
  "lop3.b32 a3, s3, 0x000F000F, 0x43004300, 0xEA;\n\t"                          \
  "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "      \
  "{a0, a1, a2, a3}, {" B0 ", " B1 "}, " CIN ";\n\t"

// The first step starts from zero (a zero register as the accumulator
// input); the four tiles a warp runs per group are independent chains.
__device__ __forceinline__ void tile_group_s(float (&d)[4], const uint4 wa, const uint4 wb,
                                             const uint4 (&x)[4]) {
  asm("{\n\t.reg .b32 a0, a1, a2, a3, s0, s1, s2, s3;\n\t"
      ".reg .f32 z;\n\tmov.b32 z, 0;\n\t"
      W4S_STEP("%4", "%8", "%12", "%13", "0", "{z, z, z, z}")
      W4S_STEP("%4", "%8", "%14", "%15", "8", "{%0, %1, %2, %3}")
      W4S_STEP("%5", "%9", "%16", "%17", "0", "{%0, %1, %2, %3}")
      W4S_STEP("%5", "%9", "%18", "%19", "8", "{%0, %1, %2, %3}")
      W4S_STEP("%6", "%10", "%20", "%21", "0", "{%0, %1, %2, %3}")
      W4S_STEP("%6", "%10", "%22", "%23", "8", "{%0, %1, %2, %3}")
      W4S_STEP("%7", "%11", "%24", "%25", "0", "{%0, %1, %2, %3}")
      W4S_STEP("%7", "%11", "%26", "%27", "8", "{%0, %1, %2, %3}")
      "}"
      : "=&f"(d[0]), "=&f"(d[1]), "=&f"(d[2]), "=&f"(d[3])
      : "r"(wa.x), "r"(wa.y), "r"(wa.z), "r"(wa.w), "r"(wb.x), "r"(wb.y), "r"(wb.z), "r"(wb.w),
        "r"(x[0].x), "r"(x[0].y), "r"(x[0].z), "r"(x[0].w), "r"(x[1].x), "r"(x[1].y), "r"(x[1].z),
        "r"(x[1].w), "r"(x[2].x), "r"(x[2].y), "r"(x[2].z), "r"(x[2].w), "r"(x[3].x), "r"(x[3].y),
        "r"(x[3].z), "r"(x[3].w));
}
#undef W4S_STEP

// W4A8: one 16-row tile over one group against int8 activations, 4 steps of
// mma.m16n8k32 (u8 codes x s8 activations, exact int32 sums).  Word j of
// each row gives two A registers by masking: low nibbles (channels 0, 4, 1,
// 5 of the word's 8) and high nibbles (2, 6, 3, 7); the activation codes are
// stored in the same channel order, so x words 2j and 2j+1 are the matching
// B registers.
#define W4A8_STEP(VA, VB, B0, B1, CIN)                                           \
  "shr.b32 s0, " VA ", 4;\n\t"                                                   \
  "shr.b32 s1, " VB ", 4;\n\t"                                                   \
  "and.b32 a0, " VA ", 0x0F0F0F0F;\n\t"                                          \
  "and.b32 a1, " VB ", 0x0F0F0F0F;\n\t"                                          \
  "and.b32 a2, s0, 0x0F0F0F0F;\n\t"                                              \
  "and.b32 a3, s1, 0x0F0F0F0F;\n\t"                                              \
  "mma.sync.aligned.m16n8k32.row.col.s32.u8.s8.s32 {%0, %1, %2, %3}, "            \
  "{a0, a1, a2, a3}, {" B0 ", " B1 "}, " CIN ";\n\t"

__device__ __forceinline__ void tile_group_a8(int (&d)[4], const uint4 wa, const uint4 wb,
                                              const uint4 (&x)[2]) {
  asm("{\n\t.reg .b32 a0, a1, a2, a3, s0, s1;\n\t"
      ".reg .s32 z;\n\tmov.b32 z, 0;\n\t"
      W4A8_STEP("%4", "%8", "%12", "%13", "{z, z, z, z}")
      W4A8_STEP("%5", "%9", "%14", "%15", "{%0, %1, %2, %3}")
      W4A8_STEP("%6", "%10", "%16", "%17", "{%0, %1, %2, %3}")
      W4A8_STEP("%7", "%11", "%18", "%19", "{%0, %1, %2, %3}")
      "}"
      : "=&r"(d[0]), "=&r"(d[1]), "=&r"(d[2]), "=&r"(d[3])
      : "r"(wa.x), "r"(wa.y), "r"(wa.z), "r"(wa.w), "r"(wb.x), "r"(wb.y), "r"(wb.z), "r"(wb.w),
        "r"(x[0].x), "r"(x[0].y), "r"(x[0].z), "r"(x[0].w), "r"(x[1].x), "r"(x[1].y),
        "r"(x[1].z), "r"(x[1].w));
}
#undef W4A8_STEP

__device__ __forceinline__ float half_bits_to_float(uint32_t h) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h)));
}

// Position of a warp in its list of units: the bundle, the linear it
// belongs to, the row block and K part this warp takes in it, and the group
// range of that part.
struct UnitPos {
  int bundle, item, ks, part, rb, g, ge;
};

// Moves p to the first bundle at or after `bundle` (stepping by the grid)
// in which this warp has a unit; p.bundle = total when there is none.
// Bundles only ever increase, so the linear is found by a forward scan.
__device__ __forceinline__ void enter_bundle(const StreamBatch& b, UnitPos& p, int bundle,
                                             int warp, int total) {
  for (; bundle < total; bundle += static_cast<int>(gridDim.x)) {
    while (b.unit_start[p.item + 1] <= bundle) ++p.item;
    const int ks = b.ks[p.item];
    const int rb = (bundle - b.unit_start[p.item]) * (kStreamWarps / ks) + warp / ks;
    if (rb * 64 < b.N[p.item]) {
      const int G = b.K[p.item] >> 7;
      p.bundle = bundle;
      p.ks = ks;
      p.part = warp % ks;
      p.rb = rb;
      p.g = p.part * G / ks;
      p.ge = (p.part + 1) * G / ks;
      return;
    }
  }
  p.bundle = total;
}

constexpr int kTiles = 4;  // 16-row mma tiles per unit (64 weight rows)
// One ring slot of a warp: [tile][row g | row g + 8][lane][16 bytes] of
// packed codes, then [tile][lane][4 bytes] holding this lane's scale or zero
// value of each tile.
constexpr uint32_t kSlotCodes = kTiles * 1024;
constexpr uint32_t kSlotBytes = kSlotCodes + kTiles * 128;

// A8 = false: bf16 activations (W4A16).  A8 = true: int8 activation codes
// with per-token scales and per-group code sums (W4A8).
template <bool SYM, int S, int MIN_CTAS, bool A8>
__global__ void __launch_bounds__(kStreamThreads, MIN_CTAS)
    gemv_w4a16_stream_kernel(const __grid_constant__ StreamBatch b, int static_weights) {
  // Partial sums of the warps of a unit: [warp][tile][lane].
  __shared__ float4 red[kStreamWarps][kTiles][32];
  extern __shared__ __align__(16) uint8_t ring_raw[];  // per warp: S slots

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2;
  const int t = lane & 3;
  const int first = static_cast<int>(blockIdx.x);
  const int stride = static_cast<int>(gridDim.x);
  const int units = b.unit_start[b.count];  // bundles of the launch
  const int M = b.M;
  const uint32_t ring = smem_u32(ring_raw) + warp * (S * kSlotBytes);

  pdl_launch_dependents();

  // ---- load side: S groups ahead of the compute side -------------------
  // Per group lane t copies 16 bytes of rows g and g + 8 of each tile, and
  // per tile the aligned 4-byte word holding t = 0: the scale of row g, 1:
  // the scale of row g + 8, 2: the zero of row g, 3: the zero of row g + 8
  // (only the value's own two bytes are read: from an even element index the
  // word's first two, from an odd one all four).  Rows beyond N copy nothing
  // (zero fill) from row 0's address.
  UnitPos lp{0, 0, 1, 0, 0, 0, 0};
  const uint8_t* lw = nullptr;   // this lane's bytes of row 16*0 + g at group lp.g
  const uint8_t* lw0 = nullptr;  // the same bytes of row 0 (source of skipped copies)
  const uint8_t* lsp[kTiles];    // per tile: the aligned word holding this lane's value
  uint32_t lsv = 0;              // bit rt: this lane's value row of tile rt in range
  uint32_t lpar = 0;             // parity of the element index of this lane's values
  size_t lrow8 = 0;              // 8 rows of codes, in bytes
  uint32_t lvalid = 0;           // bit 2*rt+h: row 16rt + 8h + g in range
  auto load_enter = [&](int bundle) {
    enter_bundle(b, lp, bundle, warp, units);
    if (lp.bundle >= units) return;
    const int K = b.K[lp.item];
    const int N = b.N[lp.item];
    const int G = K >> 7;
    const int row = lp.rb * (16 * kTiles) + g;
    const int vrow = row + 8 * (t & 1);  // the row of this lane's value
    lvalid = 0;
    lsv = 0;
#pragma unroll
    for (int rt = 0; rt < kTiles; ++rt) {
      if (row + 16 * rt < N) lvalid |= 1u << (2 * rt);
      if (row + 16 * rt + 8 < N) lvalid |= 2u << (2 * rt);
      if (vrow + 16 * rt < N && (t < 2 || !SYM)) lsv |= 1u << rt;
    }
    lrow8 = static_cast<size_t>(K) * 4;
    lw0 = b.qw[lp.item] + lp.g * 64 + 16 * t;
    lw = lw0 + static_cast<size_t>(row) * (K >> 1);
    const uint16_t* base = (t < 2 || SYM) ? b.scales[lp.item] : b.zeros[lp.item];
    const size_t e0 = static_cast<size_t>(vrow) * G + lp.g;  // tile 0 (rows 16 G apart)
    lpar = static_cast<uint32_t>(e0 & 1);
#pragma unroll
    for (int rt = 0; rt < kTiles; ++rt) {
      const size_t e = ((lsv >> rt) & 1u) ? e0 + static_cast<size_t>(16 * rt) * G
                                          : static_cast<size_t>(lp.g);
      lsp[rt] = reinterpret_cast<const uint8_t*>(base + (e & ~size_t{1}));
    }
  };
  // Requests the next group into ring slot `slot` (one commit group per
  // call, empty once the warp's list is exhausted).
  auto load_group = [&](uint32_t slot) {
    if (lp.bundle < units) {
      const uint32_t dst = ring + slot * kSlotBytes;
      if ((lvalid & 0xFFu) == 0xFFu) {  // every row of the unit in range
        const uint8_t* q = lw;
#pragma unroll
        for (int p = 0; p < 2 * kTiles; ++p, q += lrow8) cp_async16(dst + p * 512 + lane * 16, q, true);
      } else {
#pragma unroll
        for (int p = 0; p < 2 * kTiles; ++p) {
          const bool v = (lvalid >> p) & 1u;
          cp_async16(dst + p * 512 + lane * 16, v ? lw + p * lrow8 : lw0, v);
        }
      }
      const uint32_t sz = 2u << lpar;  // bytes of an in-range value word
      const uint32_t adv = lpar << 2;  // the next group's value is in the next word after an odd one
#pragma unroll
      for (int rt = 0; rt < kTiles; ++rt) {
        cp_async4_part(dst + kSlotCodes + rt * 128 + lane * 4, lsp[rt],
                       ((lsv >> rt) & 1u) ? sz : 0u);
        lsp[rt] += adv;
      }
      lpar ^= 1u;
      ++lp.g;
      lw += 64;
      lw0 += 64;
      if (lp.g == lp.ge) load_enter(lp.bundle + stride);
    }
    cp_async_commit();
  };

  load_enter(first);
  // With static weights the first groups are requested before the
  // dependency wait (they are not written by the preceding kernel).
  if (!static_weights) pdl_wait();
#pragma unroll 1
  for (int d = 0; d < S; ++d) load_group(d);
  pdl_wait();  // x is read, and y written, only after the preceding kernel

  // ---- compute side ------------------------------------------------------
  UnitPos cp{0, 0, 1, 0, 0, 0, 0};
  enter_bundle(b, cp, first, warp, units);
  // x fragments (token g, channels 32t .. 32t+31 of a group) are loaded one
  // group ahead of use; xq walks the compute list one group ahead of cp.
  // W4A8: dst[0..1] hold the 32 activation codes, dst[2].x / .y the group's
  // code sums of tokens 2t and 2t + 1 (the mma's output columns).
  // A lane whose token is beyond M reads token M - 1 instead: its mma
  // columns are never stored, so no zero fill and no predicate are needed.
  // The lane's x pointer runs on through a unit and is set at unit entry.
  UnitPos xq = cp;
  const int xtok = g < M ? g : M - 1;
  const int xt0 = 2 * t < M ? 2 * t : M - 1;
  const int xt1 = 2 * t + 1 < M ? 2 * t + 1 : M - 1;
  const uint4* xptr = nullptr;     // this lane's x chunk of group xq.g
  const int32_t* xsp0 = nullptr;   // W4A8: group code sums of tokens xt0, xt1 at group xq.g
  const int32_t* xsp1 = nullptr;
  auto x_enter = [&]() {
    if (xq.bundle >= units) return;
    const int K = b.K[xq.item];
    if constexpr (A8) {
      xptr = reinterpret_cast<const uint4*>(reinterpret_cast<const int8_t*>(b.x[xq.item]) +
                                            static_cast<size_t>(xtok) * K + xq.g * 128 + 32 * t);
      xsp0 = b.xsum[xq.item] + static_cast<size_t>(xt0) * (K >> 7) + xq.g;
      xsp1 = b.xsum[xq.item] + static_cast<size_t>(xt1) * (K >> 7) + xq.g;
    } else {
      xptr = reinterpret_cast<const uint4*>(b.x[xq.item] + static_cast<size_t>(xtok) * K +
                                            xq.g * 128 + 32 * t);
    }
  };
  auto load_x = [&](uint4 (&dst)[4]) {
    if (xq.bundle >= units) return;
    if constexpr (A8) {
      dst[0] = __ldg(xptr);
      dst[1] = __ldg(xptr + 1);
      dst[2].x = static_cast<uint32_t>(__ldg(xsp0));
      dst[2].y = static_cast<uint32_t>(__ldg(xsp1));
      xptr += 8;  // 128 int8 codes
      ++xsp0;
      ++xsp1;
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) dst[j] = __ldg(xptr + j);
      xptr += 16;  // 128 bf16 values
    }
    if (++xq.g == xq.ge) {
      enter_bundle(b, xq, xq.bundle + stride, warp, units);
      x_enter();
    }
  };
  uint4 xnext[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) xnext[j] = make_uint4(0u, 0u, 0u, 0u);
  x_enter();
  load_x(xnext);
  float acc[kTiles][4];
#pragma unroll
  for (int rt = 0; rt < kTiles; ++rt) acc[rt][0] = acc[rt][1] = acc[rt][2] = acc[rt][3] = 0.f;
  const uint32_t ones = kOnesBf16x2;
  // First row of this lane's fragment in the unit; parity of the element
  // index of its scale/zero values (the same for all tiles, 16*G apart).
  int crow = 0, cpar = 0;
  auto compute_enter = [&]() {
    const int G = b.K[cp.item] >> 7;
    crow = cp.rb * (16 * kTiles) + g;
    cpar = ((crow + 8 * (t & 1)) * G + cp.g) & 1;
  };
  if (cp.bundle < units) compute_enter();

  uint32_t slot = 0;
  const float zadd = (!SYM && t >= 2) ? 128.0f : 0.0f;
#pragma unroll 1
  while (cp.bundle < units) {
    uint4 xv[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) xv[j] = xnext[j];
    load_x(xnext);
    // W4A16: per-token sums of x over the group (all-ones rows), two chains.
    float xs[4] = {0.f, 0.f, 0.f, 0.f};
    if constexpr (!A8) {
      float xt[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        mma_16816(xs, ones, ones, ones, ones, xv[j].x, xv[j].y);
        mma_16816(xt, ones, ones, ones, ones, xv[j].z, xv[j].w);
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) xs[k] += xt[k];
    }
    // This slot's copies (issued S groups ago) have landed; every lane reads
    // back only what it copied itself.
    cp_async_wait<S - 1>();
    const uint32_t src = ring + slot * kSlotBytes;
    const int sh = 16 * cpar;
    const uint32_t hsel = cpar ? 0x3232u : 0x3210u;  // the value's half into the low 16 bits
#pragma unroll
    for (int rt = 0; rt < kTiles; ++rt) {
      const uint4 wa = lds128s(src + rt * 1024 + lane * 16);
      const uint4 wb = lds128s(src + rt * 1024 + 512 + lane * 16);
      const uint32_t wv = lds32s(src + kSlotCodes + rt * 128 + lane * 4);
      const int q0 = lane & ~3;
      if constexpr (A8) {
        const uint32_t v = (wv >> sh) & 0xFFFFu;
        const float sa = half_bits_to_float(__shfl_sync(0xffffffffu, v, q0 + 0));
        const float sb = half_bits_to_float(__shfl_sync(0xffffffffu, v, q0 + 1));
        // D = sum (q - z) x8 = sum q x8 - z * S (exact int32), then scale.
        int c[4];
        const uint4 x8[2] = {xv[0], xv[1]};
        tile_group_a8(c, wa, wb, x8);
        int za = 8, zb = 8;  // symmetric: zero 8
        if (!SYM) {
          za = __float2int_rn(half_bits_to_float(__shfl_sync(0xffffffffu, v, q0 + 2)));
          zb = __float2int_rn(half_bits_to_float(__shfl_sync(0xffffffffu, v, q0 + 3)));
        }
        const int s0 = static_cast<int>(xv[2].x), s1 = static_cast<int>(xv[2].y);
        acc[rt][0] = fmaf(sa, __int2float_rn(c[0] - za * s0), acc[rt][0]);
        acc[rt][1] = fmaf(sa, __int2float_rn(c[1] - za * s1), acc[rt][1]);
        acc[rt][2] = fmaf(sb, __int2float_rn(c[2] - zb * s0), acc[rt][2]);
        acc[rt][3] = fmaf(sb, __int2float_rn(c[3] - zb * s1), acc[rt][3]);
      } else {
        // Each lane widens its own value once (a zero lane adds 128); the
        // shuffles then move finished floats.
        const float fv = half_bits_to_float(__byte_perm(wv, 0u, hsel) & 0xFFFFu) + zadd;
        const float sa = __shfl_sync(0xffffffffu, fv, q0 + 0);
        const float sb = __shfl_sync(0xffffffffu, fv, q0 + 1);
        float c[4];
        tile_group_s(c, wa, wb, xv);
        float za = 136.0f, zb = 136.0f;  // 128 + zero (symmetric: zero 8)
        if (!SYM) {
          za = __shfl_sync(0xffffffffu, fv, q0 + 2);
          zb = __shfl_sync(0xffffffffu, fv, q0 + 3);
        }
        acc[rt][0] = fmaf(sa, fmaf(-za, xs[0], c[0]), acc[rt][0]);
        acc[rt][1] = fmaf(sa, fmaf(-za, xs[1], c[1]), acc[rt][1]);
        acc[rt][2] = fmaf(sb, fmaf(-zb, xs[2], c[2]), acc[rt][2]);
        acc[rt][3] = fmaf(sb, fmaf(-zb, xs[3], c[3]), acc[rt][3]);
      }
    }
    // The slot's data has been consumed: refill it with the group S ahead.
    load_group(slot);
    slot = slot + 1 == S ? 0 : slot + 1;
    cpar ^= 1;

    if (++cp.g == cp.ge) {
      // End of the unit: reduce over its ks warps (fixed order), store.
      if (cp.ks > 1) {
        // Named barrier of the row block's ks warps; the ids of ks = 2 (1, 2)
        // and ks = 4 (3) differ, so warps in different bundles never meet
        // on one barrier with different counts.
        const int bar_id = cp.ks == 2 ? 1 + (warp >> 1) : 3;
        const int bar_n = 32 * cp.ks;
        if (cp.part > 0) {
#pragma unroll
          for (int rt = 0; rt < kTiles; ++rt)
            red[warp][rt][lane] = make_float4(acc[rt][0], acc[rt][1], acc[rt][2], acc[rt][3]);
        }
        asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(bar_n) : "memory");
        if (cp.part == 0) {
          for (int p = 1; p < cp.ks; ++p) {
#pragma unroll
            for (int rt = 0; rt < kTiles; ++rt) {
              const float4 r = red[warp + p][rt][lane];
              acc[rt][0] += r.x;
              acc[rt][1] += r.y;
              acc[rt][2] += r.z;
              acc[rt][3] += r.w;
            }
          }
        }
        // The buffer is free again only once the first warp has read it.
        asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(bar_n) : "memory");
      }
      if (cp.part == 0) {
        const int N = b.N[cp.item];
        __nv_bfloat16* y = b.y[cp.item];
        const int m0 = 2 * t, m1 = 2 * t + 1;
        if constexpr (A8) {  // y = xscale_m * sum_g scale * D
          const float* xsc = b.xscale[cp.item];
          const float f0 = m0 < M ? __ldg(xsc + m0) : 0.f;
          const float f1 = m1 < M ? __ldg(xsc + m1) : 0.f;
#pragma unroll
          for (int rt = 0; rt < kTiles; ++rt) {
            acc[rt][0] *= f0;
            acc[rt][1] *= f1;
            acc[rt][2] *= f0;
            acc[rt][3] *= f1;
          }
        }
#pragma unroll
        for (int rt = 0; rt < kTiles; ++rt) {
          const int r0 = crow + 16 * rt;
          if (r0 < N) {
            if (m0 < M) y[static_cast<size_t>(m0) * N + r0] = __float2bfloat16_rn(acc[rt][0]);
            if (m1 < M) y[static_cast<size_t>(m1) * N + r0] = __float2bfloat16_rn(acc[rt][1]);
          }
          if (r0 + 8 < N) {
            if (m0 < M) y[static_cast<size_t>(m0) * N + r0 + 8] = __float2bfloat16_rn(acc[rt][2]);
            if (m1 < M) y[static_cast<size_t>(m1) * N + r0 + 8] = __float2bfloat16_rn(acc[rt][3]);
          }
        }
      }
#pragma unroll
      for (int rt = 0; rt < kTiles; ++rt) acc[rt][0] = acc[rt][1] = acc[rt][2] = acc[rt][3] = 0.f;
      enter_bundle(b, cp, cp.bundle + stride, warp, units);
      if (cp.bundle < units) compute_enter();
    }
  }
  cp_async_wait<0>();  // no copy may still target shared memory at exit
}

// Two ring depths: 3 slots per warp with three CTAs per SM for launches with
// many bundles per SM (the warps' streams continue across units), and 5 slots
// with two CTAs per SM for launches of at most two bundles per SM, whose
// warps see one short unit each and need more bytes in flight from the start.
constexpr int kDepthWide = 3;
constexpr int kDepthDeep = 5;

template <int S>
constexpr size_t ring_bytes() {
  return static_cast<size_t>(kStreamWarps) * S * kSlotBytes;
}

// Resident CTAs per SM of one kernel instance (opted in to its shared memory
// once per device).
template <auto kern, size_t kBytes>
cudaError_t stream_occupancy(int dev, int* occ) {
  static int per_sm[64] = {};
  int o = dev < 64 ? __atomic_load_n(&per_sm[dev], __ATOMIC_ACQUIRE) : 0;
  if (o == 0) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kBytes));
    if (e != cudaSuccess) return e;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, kern, kStreamThreads, kBytes);
    if (e != cudaSuccess) return e;
    if (o < 1) o = 1;
    if (dev < 64) __atomic_store_n(&per_sm[dev], o, __ATOMIC_RELEASE);
  }
  *occ = o;
  return cudaSuccess;
}

// A launch with few row blocks splits K further (up to 4 parts of at least
// 2 groups) while that at most doubles its bundles within `slots` CTAs, so
// that small launches still spread over the SMs.
void plan_splits(StreamBatch& b, int slots) {
  for (;;) {
    int more = 0;
    for (int i = 0; i < b.count; ++i)
      if (b.ks[i] < 4 && b.K[i] / 128 / (2 * b.ks[i]) >= 2) ++more;
    if (more == 0 || 2LL * b.unit_start[b.count] > slots) break;
    for (int i = 0; i < b.count; ++i) {
      if (b.ks[i] < 4 && b.K[i] / 128 / (2 * b.ks[i]) >= 2) b.ks[i] *= 2;
      const int per = kStreamWarps / b.ks[i];
      b.unit_start[i + 1] = b.unit_start[i] + ((b.N[i] + 63) / 64 + per - 1) / per;
    }
  }
}

template <auto kern, size_t kBytes>
cudaError_t launch_stream_cfg(const StreamBatch& b, int grid, bool pdl, bool static_w,
                              cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kStreamThreads, 1, 1);
  cfg.dynamicSmemBytes = kBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  if (pdl) {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
  }
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, b, static_cast<int>(pdl && static_w));
}

template <bool SYM, bool A8>
cudaError_t launch_stream_t(StreamBatch& b, bool pdl, bool static_w, cudaStream_t stream,
                            int num_sms) {
  constexpr auto kWide = gemv_w4a16_stream_kernel<SYM, kDepthWide, 3, A8>;
  constexpr auto kDeep = gemv_w4a16_stream_kernel<SYM, kDepthDeep, 2, A8>;
  constexpr size_t kWideBytes = ring_bytes<kDepthWide>();
  constexpr size_t kDeepBytes = ring_bytes<kDepthDeep>();
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int occ_wide = 0, occ_deep = 0;
  e = stream_occupancy<kWide, kWideBytes>(dev, &occ_wide);
  if (e != cudaSuccess) return e;
  e = stream_occupancy<kDeep, kDeepBytes>(dev, &occ_deep);
  if (e != cudaSuccess) return e;
  plan_splits(b, num_sms * occ_wide);
  const int bundles = b.unit_start[b.count];
  if (bundles <= num_sms * occ_deep)
    return launch_stream_cfg<kDeep, kDeepBytes>(b, bundles, pdl, static_w, stream);
  const int slots = num_sms * occ_wide;
  return launch_stream_cfg<kWide, kWideBytes>(b, bundles < slots ? bundles : slots, pdl,
                                                static_w, stream);
}

}  // namespace

// Splits K so that a warp's part has at most 16 groups where it can (at
// most 4 parts, each of at least 2 groups): units of similar length keep the
// warps' totals even when linears of different K share a launch.
void stream_batch_add(StreamBatch& b, const void* x, const int32_t* qw, const uint16_t* sc,
                      const uint16_t* z, int N, int K, void* y, const int32_t* xsum,
                      const float* xscale) {
  const int i = b.count;
  b.x[i] = static_cast<const __nv_bfloat16*>(x);
  b.xsum[i] = xsum;
  b.xscale[i] = xscale;
  b.qw[i] = reinterpret_cast<const uint8_t*>(qw);
  b.scales[i] = sc;
  b.zeros[i] = z;
  b.y[i] = static_cast<__nv_bfloat16*>(y);
  b.N[i] = N;
  b.K[i] = K;
  const int G = K / 128;
  int ks = 1;
  while (ks < 4 && (G + ks - 1) / ks > 16 && G / (2 * ks) >= 2) ks *= 2;
  b.ks[i] = ks;
  const int row_blocks = (N + 63) / 64;
  const int per = kStreamWarps / ks;  // row blocks per bundle
  b.unit_start[i + 1] = b.unit_start[i] + (row_blocks + per - 1) / per;
  b.count = i + 1;
}

template <bool SYM>
cudaError_t plan_stream_t(StreamBatch& b, int num_sms, int* bundles) {
  constexpr auto kWide = gemv_w4a16_stream_kernel<SYM, kDepthWide, 3, false>;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  int occ = 0;
  e = stream_occupancy<kWide, ring_bytes<kDepthWide>()>(dev, &occ);
  if (e != cudaSuccess) return e;
  plan_splits(b, num_sms * occ);
  *bundles = b.unit_start[b.count];
  return cudaSuccess;
}

cudaError_t plan_gemv_stream(StreamBatch& b, bool symmetric, int num_sms, int* bundles) {
  return symmetric ? plan_stream_t<true>(b, num_sms, bundles)
                   : plan_stream_t<false>(b, num_sms, bundles);
}

cudaError_t launch_gemv_stream(StreamBatch& b, bool symmetric, bool pdl, bool static_w,
                               cudaStream_t stream, int num_sms) {
  if (b.count < 1 || b.M < 1 || b.M > 8) return cudaErrorInvalidValue;
  if (b.a8)
    return symmetric ? launch_stream_t<true, true>(b, pdl, static_w, stream, num_sms)
                     : launch_stream_t<false, true>(b, pdl, static_w, stream, num_sms);
  return symmetric ? launch_stream_t<true, false>(b, pdl, static_w, stream, num_sms)
                   : launch_stream_t<false, false>(b, pdl, static_w, stream, num_sms);
}

}  // namespace w4
