// Decode W4A16 GEMV, tensor-map kernel: y[M, N] = x[M, K] . dequant(Wq)^T for
// M <= 16 (up to 64 with W4_LINEAR_FORCE_GEMV, in chunks of 16 tokens).
// HBM-bound on the packed weight stream (0.53125 B/weight asymmetric,
// 0.515625 symmetric).  It serves 9 <= M <= 64 and decode launches too small
// for the persistent streaming kernel (gemv_stream.cu), which it beats there
// because its cluster K split fills the GPU with few rows.
//
// A CTA owns 64 weight rows and one K slice (the K dimension is split over
// the CTAs of a thread-block cluster).  One producer thread streams the
// slice through a ring of shared-memory stages with TMA, one 128-channel
// group per stage: the 64 x 64-byte tile of packed codes plus the matching
// x tile (tokens x 128 channels, 128-byte swizzled).  Four consumer warps
// take the groups in turn; for its group a warp turns all four 16-row tiles
// into exact bf16 values 128 + q in registers (one mask/OR per pair of codes:
// the canonical nibble order puts adjacent channels in nibbles i and i+4),
// runs mma.m16n8k16 against the x fragments (rows = weights, columns =
// tokens), removes (128 + zero) * sum_k x_k with one extra mma of all-ones
// rows per group (shared by the four tiles) and adds scale * result to fp32
// accumulators.  Partial sums are reduced across the four warps in shared
// memory and across the cluster in rank order through distributed shared
// memory (no global scratch; deterministic).
//
// Inside one group the mma's 16 reduction slots map to channels as follows:
// lane t (= lane % 4) covers channels 32t..32t+31 of the group and step s
// (0..7) uses channels 32t+4s..32t+4s+3, so the x operand of step s is two
// consecutive bf16 pairs and needs no permutation.
//
// Every wait is bounded; a CTA that gives up records it in the device error
// word, drains its own TMA loads and returns.  Every TMA load feeds only its
// own CTA.
#include <cooperative_groups.h>
#include <cudaTypedefs.h>

#include "w4_common.cuh"
#include "w4_kernels.h"

namespace cg = cooperative_groups;

namespace w4 {

namespace {

constexpr int kRows = 64;                 // weight rows per CTA
constexpr int kConsumerWarps = 4;
constexpr int kThreads = 32 * (kConsumerWarps + 1);
constexpr int kMaxSliceGroups = 80;       // groups per CTA slice (scale table)
constexpr uint32_t kOnes = 0x3F803F80u;    // bf16x2 (1.0, 1.0)
constexpr uint32_t kWTileBytes = kRows * 64;
constexpr unsigned kKernelIdGemv = 1;

// Shared-memory layout of one CTA (identical on host and device).  The
// ring holds min(max stages, groups of the slice) stages, so small slices
// leave room for more CTAs per SM (and for the next kernel under PDL).
struct GemvLayout {
  uint32_t x_half, stage, ring, sz, red, part, bars, misc, total;
  int stages;
};

__host__ __device__ inline GemvLayout gemv_layout(int nt, int gs_max) {
  GemvLayout L;
  const int tokens = 8 * nt;
  L.x_half = tokens * 128;                      // tokens x 64 channels, bf16
  // Up to 8 tokens the stages hold weights only (consumers read x from
  // global memory, where it stays cached), six per consumer warp; 16 tokens
  // take the x tile through the stage as well, two stages per warp.  Stage s
  // is only ever consumed by warp s % 4 (the ring length is a multiple of the
  // warp count whenever a stage is reused).
  L.stage = nt == 1 ? kWTileBytes : kWTileBytes + 2 * L.x_half;  // multiple of 1024
  const int max_stages = (nt == 1 ? 6 : 2) * kConsumerWarps;
  L.stages = gs_max < max_stages ? (gs_max < 1 ? 1 : gs_max) : max_stages;
  L.ring = 0;
  // Scale table [64][gs_max | 1] (scale | zero << 16): an odd row pitch puts
  // the eight rows that one epilogue read touches in distinct banks.
  L.sz = L.ring + L.stages * L.stage;
  // The per-warp partial sums reuse the ring once every stage is consumed.
  L.red = L.ring;                                // [4][tokens][64] f32
  const uint32_t red_end = L.red + kConsumerWarps * tokens * kRows * 4;
  L.part = L.sz + ((kRows * (gs_max | 1) * 4 + 15) & ~15u);  // [tokens][64] f32
  if (L.part < red_end) L.part = red_end;
  L.bars = L.part + tokens * kRows * 4;          // full[S], empty[S]
  L.misc = L.bars + 2 * L.stages * 8;
  L.total = L.misc + 16 + 1024;                  // + alignment slack
  return L;
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 r;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "r"(addr));
  return r;
}

// One reduction step of one 16-row tile, fused so that the code pairs land
// directly in the mma's operand registers: for the two packed words va (row
// g) and vb (row g+8), shifted right by SH, the A fragment is
//   (x >> SH) & 0x000F000F | 0x43004300   and   (x >> (SH+4)) & ...,
// i.e. bf16x2 (128 + q) pairs of adjacent channels (exact: bf16 has unit
// spacing on [128, 256)).
// One 16-row tile over one 128-channel group, 8 reduction steps, in a single
// asm block: the code pairs and the running accumulator stay in registers the
// block owns.  Word j of each row (channels 8j..8j+7 of this lane's 32) feeds
// steps 2j (pairs at shift 0 and 4) and 2j+1 (shift 8 and 12); the A fragment
// of a step is (w >> sh) & 0x000F000F | 0x43004300, bf16x2 (128 + q) pairs of
// adjacent channels (exact: bf16 has unit spacing on [128, 256)).
// x0..x3: this lane's x fragments (channels 8j..8j+7 as four bf16x2).
#define W4_TILE_STEP(VA, VB, B0, B1, SH0)                                       \
  "shr.b32 s0, " VA ", " SH0 ";\n\t"                                            \
  "shr.b32 s1, " VB ", " SH0 ";\n\t"                                            \
  "shr.b32 s2, " VA ", " SH0 "+4;\n\t"                                          \
  "shr.b32 s3, " VB ", " SH0 "+4;\n\t"                                          \
  "lop3.b32 a0, s0, 0x000F000F, 0x43004300, 0xEA;\n\t"                          \
  "lop3.b32 a1, s1, 0x000F000F, 0x43004300, 0xEA;\n\t"                          \
  "lop3.b32 a2, s2, 0x000F000F, 0x43004300, 0xEA;\n\t"                          \
  "lop3.b32 a3, s3, 0x000F000F, 0x43004300, 0xEA;\n\t"                          \
  "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {c0, c1, c2, c3}, "      \
  "{a0, a1, a2, a3}, {" B0 ", " B1 "}, {c0, c1, c2, c3};\n\t"

__device__ __forceinline__ void tile_group(float (&d)[4], const uint4 wa, const uint4 wb,
                                           const uint4 (&x)[4]) {
  asm("{\n\t.reg .b32 a0, a1, a2, a3, s0, s1, s2, s3;\n\t"
      ".reg .f32 c0, c1, c2, c3;\n\t"
      "mov.b32 c0, 0;\n\tmov.b32 c1, 0;\n\tmov.b32 c2, 0;\n\tmov.b32 c3, 0;\n\t"
      W4_TILE_STEP("%4", "%8", "%12", "%13", "0")
      W4_TILE_STEP("%4", "%8", "%14", "%15", "8")
      W4_TILE_STEP("%5", "%9", "%16", "%17", "0")
      W4_TILE_STEP("%5", "%9", "%18", "%19", "8")
      W4_TILE_STEP("%6", "%10", "%20", "%21", "0")
      W4_TILE_STEP("%6", "%10", "%22", "%23", "8")
      W4_TILE_STEP("%7", "%11", "%24", "%25", "0")
      W4_TILE_STEP("%7", "%11", "%26", "%27", "8")
      "mov.b32 %0, c0;\n\tmov.b32 %1, c1;\n\tmov.b32 %2, c2;\n\tmov.b32 %3, c3;\n\t}"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(wa.x), "r"(wa.y), "r"(wa.z), "r"(wa.w), "r"(wb.x), "r"(wb.y), "r"(wb.z), "r"(wb.w),
        "r"(x[0].x), "r"(x[0].y), "r"(x[0].z), "r"(x[0].w), "r"(x[1].x), "r"(x[1].y), "r"(x[1].z),
        "r"(x[1].w), "r"(x[2].x), "r"(x[2].y), "r"(x[2].z), "r"(x[2].w), "r"(x[3].x), "r"(x[3].y),
        "r"(x[3].z), "r"(x[3].w));
}
#undef W4_TILE_STEP

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}


__device__ __forceinline__ void named_bar_consumers() {
  asm volatile("bar.sync 1, %0;" ::"n"(32 * kConsumerWarps) : "memory");
}

template <int NT, bool SYM>
__global__ void __launch_bounds__(kThreads, 2)
    gemv_w4a16_kernel(const __grid_constant__ GemvBatch b, int static_weights, unsigned* err) {
  constexpr int kTokens = 8 * NT;
  // This CTA's linear of the batch and its 64-row block.
  int item = 0;
  {
    int lo = 0, hi = b.count - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (b.cta_start[mid] <= static_cast<int>(blockIdx.x)) lo = mid; else hi = mid - 1;
    }
    item = lo;
  }
  const CUtensorMap* tmap_w = &b.tw[item];   // uint8 [N, K/2], box 64 x 64
  const CUtensorMap* tmap_x = &b.tx[item];   // bf16 [M, K], box 64 x tokens, SW128
  const uint16_t* __restrict__ scales = b.scales[item];
  const uint16_t* __restrict__ zeros = b.zeros[item];
  __nv_bfloat16* __restrict__ y = b.y[item];
  const int M = b.M, N = b.N[item], K = b.K[item], ksplit = b.ksplit, gs_max = b.gs_max;
  const GemvLayout L = gemv_layout(NT, gs_max);
  const int S = L.stages;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* bp = smem_raw + (base - raw_addr);
  uint32_t* s_sz = reinterpret_cast<uint32_t*>(bp + L.sz);
  float* red = reinterpret_cast<float*>(bp + L.red);
  float* part = reinterpret_cast<float*>(bp + L.part);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bp + L.misc);
  const uint32_t bar0 = base + L.bars;
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (S + s); };

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = K >> 7;
  const int row0 = (static_cast<int>(blockIdx.x) - b.cta_start[item]) * kRows;
  const int rank = blockIdx.y;
  const int g_per = (G + ksplit - 1) / ksplit;
  const int g_begin = min(G, rank * g_per);
  const int gs = min(G, g_begin + g_per) - g_begin;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // Dependents may launch now: their weight prefetch overlaps this kernel.
  pdl_launch_dependents();

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------- producer ----
    // Lane w < 4 feeds consumer warp w: it refills only the stages that warp
    // reads (s = w, w + 4, ...), so a slow warp never holds back the others'
    // loads.
    if (lane < kConsumerWarps) {
      if (lane == 0) {
        tma_prefetch_desc(tmap_w);
        if (NT == 2) tma_prefetch_desc(tmap_x);
      }
      __syncwarp(0xFu);
      const uint32_t stage_tx = L.stage;
      // Stages whose weight tile was issued before the dependency wait.
      const int pre = static_weights ? min(gs, S) : 0;
      for (int i = lane; i < pre; i += kConsumerWarps) {
        const uint32_t st = base + L.ring + i * L.stage;
        mbar_arrive_expect_tx(full(i), stage_tx);
        tma_load_2d(st, tmap_w, (g_begin + i) * 64, row0, full(i));
      }
      pdl_wait();
      int issued = 0;  // groups this lane has issued (its last is issued - 1 ... )
      int last = -1;
      for (int i = lane; i < gs; i += kConsumerWarps) {
        const int s = i % S;
        const uint32_t st = base + L.ring + s * L.stage;
        const int gr = g_begin + i;
        if (i >= pre) {
          if (!mbar_wait(empty(s), ((i / S) & 1u) ^ 1u, abort_flag, err, kKernelIdGemv))
            break;
          mbar_arrive_expect_tx(full(s), stage_tx);
          tma_load_2d(st, tmap_w, gr * 64, row0, full(s));
        }
        if (NT == 2) {
          tma_load_2d(st + kWTileBytes, tmap_x, gr * 128, 0, full(s));
          tma_load_2d(st + kWTileBytes + L.x_half, tmap_x, gr * 128 + 64, 0, full(s));
        }
        last = i;
        ++issued;
      }
      if (*abort_flag) {  // drain this lane's own loads before leaving
        for (int i = last; i >= 0 && i > last - S; i -= kConsumerWarps) {
          volatile int dummy = 0;
          mbar_wait(full(i % S), (i / S) & 1u, &dummy, err, kKernelIdGemv, kWaitLimitNs / 4);
        }
      }
      (void)issued;
    }
  } else {
    // ------------------------------------------------------- consumers ---
    const int g = lane >> 2;
    const int t = lane & 3;
    // (scale | zero << 16) of this CTA's rows and groups into shared memory.
    // Thread j owns row j / 2 and every other group of it; all its loads are
    // issued before any is used, so the table costs one memory latency.
    if (!static_weights) pdl_wait();
    if (threadIdx.x < 2 * kRows) {
      const int r = threadIdx.x >> 1;
      const int row = row0 + r;
      const bool rv = row < N;
      const size_t gbase = static_cast<size_t>(rv ? row : 0) * G + g_begin;
      for (int q0 = 0; q0 < gs; q0 += 20) {
        uint32_t sv[10], zv[10];
#pragma unroll
        for (int j = 0; j < 10; ++j) {
          const int q = q0 + 2 * j + (threadIdx.x & 1);
          sv[j] = 0u;
          zv[j] = 0x4800u;  // zero 8 (symmetric)
          if (rv && q < gs) {
            sv[j] = __ldg(scales + gbase + q);
            if (!SYM) zv[j] = __ldg(zeros + gbase + q);
          }
        }
#pragma unroll
        for (int j = 0; j < 10; ++j) {
          const int q = q0 + 2 * j + (threadIdx.x & 1);
          if (q < gs) s_sz[r * (gs_max | 1) + q] = sv[j] | (zv[j] << 16);
        }
      }
    }
    named_bar_consumers();

    float acc[4][NT][4];
#pragma unroll
    for (int rt = 0; rt < 4; ++rt)
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[rt][n][i] = 0.f;

    // Up to 8 tokens: this lane's x fragment of group i (token g, channels
    // 32t .. 32t+31 of the group) comes straight from global memory, loaded
    // one group ahead; tokens beyond M are zero.
    const __nv_bfloat16* __restrict__ xg = b.xp[item];
    auto load_xg = [&](int i, uint4 (&dst)[4]) {
#pragma unroll
      for (int j = 0; j < 4; ++j) dst[j] = make_uint4(0u, 0u, 0u, 0u);
      if (g < M && i < gs) {
        const uint4* p = reinterpret_cast<const uint4*>(
            xg + static_cast<size_t>(g) * K + static_cast<size_t>(g_begin + i) * 128 + 32 * t);
#pragma unroll
        for (int j = 0; j < 4; ++j) dst[j] = __ldg(p + j);
      }
    };
    // x may be written by the preceding kernel: wait for it before the first
    // direct read (a no-op without programmatic dependent launch).
    pdl_wait();
    uint4 xnext[4];
    if (NT == 1) load_xg(warp, xnext);

    for (int i = warp; i < gs; i += kConsumerWarps) {
      const int s = i % S;
      if (!mbar_wait(full(s), (i / S) & 1u, abort_flag, err, kKernelIdGemv)) break;
      const uint32_t st = base + L.ring + s * L.stage;
      // x fragments: token 8n + g, channels 32t + 8j .. +7.
      uint4 xv[NT][4];
      if (NT == 1) {
#pragma unroll
        for (int j = 0; j < 4; ++j) xv[0][j] = xnext[j];
        load_xg(i + kConsumerWarps, xnext);
      } else {
        // 16 tokens: from the stage's two 128B-swizzled halves.
#pragma unroll
        for (int n = 0; n < NT; ++n)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t c = 4 * (t & 1) + j;
            xv[n][j] = lds128(st + kWTileBytes + (t >> 1) * L.x_half + (8 * n + g) * 128 +
                              ((c ^ g) << 4));
          }
      }
      uint4 wv[4][2];
#pragma unroll
      for (int rt = 0; rt < 4; ++rt) {
        wv[rt][0] = lds128(st + (16 * rt + g) * 64 + 16 * t);
        wv[rt][1] = lds128(st + (16 * rt + g + 8) * 64 + 16 * t);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty(s));  // the stage's data is in registers
      // Per-token sums of x over the group (an mma against all-ones rows):
      // sum_k (q - z) x_k = sum_k (128 + q) x_k - (128 + z) sum_k x_k.
      // Reduction steps outermost, tiles innermost: consecutive mmas belong
      // to independent accumulator chains.
      float xs[NT][4];
      float c[4][NT][4];
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int k = 0; k < 4; ++k) xs[n][k] = 0.f;
      const uint32_t ones[4] = {kOnes, kOnes, kOnes, kOnes};
#pragma unroll
      for (int sp = 0; sp < 8; ++sp)
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          const uint4 xx = xv[n][sp >> 1];
          mma_bf16_16816(xs[n], ones, (sp & 1) ? xx.z : xx.x, (sp & 1) ? xx.w : xx.y);
        }
#pragma unroll
      for (int rt = 0; rt < 4; ++rt)
#pragma unroll
        for (int n = 0; n < NT; ++n) tile_group(c[rt][n], wv[rt][0], wv[rt][1], xv[n]);
#pragma unroll
      for (int rt = 0; rt < 4; ++rt) {
        const uint32_t sza = s_sz[(16 * rt + g) * (gs_max | 1) + i];
        const uint32_t szb = s_sz[(16 * rt + g + 8) * (gs_max | 1) + i];
        const float sa = __half2float(__ushort_as_half(static_cast<uint16_t>(sza & 0xFFFFu)));
        const float sb = __half2float(__ushort_as_half(static_cast<uint16_t>(szb & 0xFFFFu)));
        const float za = 128.0f + __half2float(__ushort_as_half(static_cast<uint16_t>(sza >> 16)));
        const float zb = 128.0f + __half2float(__ushort_as_half(static_cast<uint16_t>(szb >> 16)));
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          acc[rt][n][0] = fmaf(sa, fmaf(-za, xs[n][0], c[rt][n][0]), acc[rt][n][0]);
          acc[rt][n][1] = fmaf(sa, fmaf(-za, xs[n][1], c[rt][n][1]), acc[rt][n][1]);
          acc[rt][n][2] = fmaf(sb, fmaf(-zb, xs[n][2], c[rt][n][2]), acc[rt][n][2]);
          acc[rt][n][3] = fmaf(sb, fmaf(-zb, xs[n][3], c[rt][n][3]), acc[rt][n][3]);
        }
      }
    }
    pdl_wait();  // (no-op when already satisfied) before this CTA writes y
    // This warp's partial sums: token 8n + 2t + {0,1}, rows 16rt + g (+8).
    // (The ring is free: every issued stage has been consumed; after a
    // timeout the results are undefined anyway.)
    named_bar_consumers();
    float* rw = red + warp * kTokens * kRows;
#pragma unroll
    for (int rt = 0; rt < 4; ++rt)
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        const int r = 16 * rt + g;
        rw[(8 * n + 2 * t) * kRows + r] = acc[rt][n][0];
        rw[(8 * n + 2 * t + 1) * kRows + r] = acc[rt][n][1];
        rw[(8 * n + 2 * t) * kRows + r + 8] = acc[rt][n][2];
        rw[(8 * n + 2 * t + 1) * kRows + r + 8] = acc[rt][n][3];
      }
    named_bar_consumers();
    for (int e = threadIdx.x; e < kTokens * kRows; e += 32 * kConsumerWarps)
    {
      float sum = 0.f;
#pragma unroll
      for (int q = 0; q < kConsumerWarps; ++q) sum += red[q * kTokens * kRows + e];
      part[e] = sum;
    }
  }

  if (ksplit > 1) {
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    if (rank == 0 && warp < kConsumerWarps && !*abort_flag) {
      for (int e = threadIdx.x; e < kTokens * kRows; e += 32 * kConsumerWarps) {
        const int m = e / kRows;
        const int r = e % kRows;
        float sum = 0.f;
        for (int q = 0; q < ksplit; ++q) sum += cluster.map_shared_rank(part, q)[e];
        const int n_out = row0 + r;
        if (m < M && n_out < N) y[static_cast<size_t>(m) * N + n_out] = __float2bfloat16_rn(sum);
      }
    }
    cluster.sync();  // peers keep their shared memory alive until rank 0 is done
  } else {
    __syncthreads();
    if (warp < kConsumerWarps && !*abort_flag) {
      for (int e = threadIdx.x; e < kTokens * kRows; e += 32 * kConsumerWarps) {
        const int m = e / kRows;
        const int r = e % kRows;
        const int n_out = row0 + r;
        if (m < M && n_out < N) y[static_cast<size_t>(m) * N + n_out] = __float2bfloat16_rn(part[e]);
      }
    }
  }
}

CUresult encode_2d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t inner,
                   uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                   CUtensorMapSwizzle swz) {
  static PFN_cuTensorMapEncodeTiled fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !p)
      return CUDA_ERROR_NOT_FOUND;
    fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled>(p);
  }
  const uint64_t dims[2] = {inner, outer};
  const uint64_t strides[1] = {row_bytes};
  const uint32_t box[2] = {box_inner, box_outer};
  const uint32_t estr[2] = {1, 1};
  return fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

template <int NT, bool SYM>
cudaError_t launch_gemv_batch_t(GemvBatch& b, bool pdl, bool static_w, cudaStream_t stream,
                                int num_sms, unsigned* err) {
  auto kern = gemv_w4a16_kernel<NT, SYM>;
  // Opt in once per device to the largest layout this kernel can use, and
  // record how many CTAs of it an SM holds.
  static unsigned long long attr_done = 0;  // bit d: device d
  static int per_sm[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !(__atomic_load_n(&attr_done, __ATOMIC_ACQUIRE) & (1ull << dev))) {
    const int max_smem = static_cast<int>(gemv_layout(NT, kMaxSliceGroups).total);
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, max_smem);
    if (e != cudaSuccess) return e;
    int nb = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern, kThreads, max_smem);
    if (e != cudaSuccess) return e;
    if (dev < 64) {
      per_sm[dev] = nb < 1 ? 1 : nb;
      __atomic_fetch_or(&attr_done, 1ull << dev, __ATOMIC_RELEASE);
    }
  }
  const int capacity = num_sms * (dev < 64 ? per_sm[dev] : 1);
  // Split K over a cluster as far as the grid still fits in one wave and
  // every CTA of every linear keeps at least two groups; a CTA's K slice
  // must fit the shared scale table.
  const int row_blocks = b.cta_start[b.count];
  int g_min = 1 << 30, g_max = 0;
  for (int i = 0; i < b.count; ++i) {
    g_min = b.K[i] / 128 < g_min ? b.K[i] / 128 : g_min;
    g_max = b.K[i] / 128 > g_max ? b.K[i] / 128 : g_max;
  }
  // Resident CTAs per SM for a given layout (its shared memory depends on the
  // slice), cached per device and layout size.
  static uint32_t occ_total[64][4] = {};
  static int occ_blocks[64][4] = {};
  auto resident = [&](uint32_t total, int& out) -> cudaError_t {
    if (dev < 64)
      for (int j = 0; j < 4; ++j)
        if (occ_total[dev][j] == total) {
          out = occ_blocks[dev][j] * num_sms;
          return cudaSuccess;
        }
    int nb = 0;
    const cudaError_t r = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kern, kThreads, total);
    if (r != cudaSuccess) return r;
    if (dev < 64) {
      int j = 0;
      while (j < 3 && occ_total[dev][j] != 0) ++j;
      occ_total[dev][j] = total;
      occ_blocks[dev][j] = nb;
    }
    out = nb * num_sms;
    return cudaSuccess;
  };
  // The largest split (1..8) whose grid still fits in one wave, with every
  // rank keeping at least two groups and a slice within the scale table.
  int ks = 1;
  for (int cand = 8; cand > 1; --cand) {
    const int gs = (g_max + cand - 1) / cand;
    if (g_min / cand < 2 || gs > kMaxSliceGroups) continue;
    int cap = 0;
    e = resident(gemv_layout(NT, gs).total, cap);
    if (e != cudaSuccess) return e;
    if (row_blocks * cand <= cap) {
      ks = cand;
      break;
    }
  }
  while ((g_max + ks - 1) / ks > kMaxSliceGroups && ks < 8) ++ks;
  if ((g_max + ks - 1) / ks > kMaxSliceGroups) return cudaErrorInvalidValue;
  (void)capacity;
  b.ksplit = ks;
  b.gs_max = (g_max + ks - 1) / ks;
  const GemvLayout L = gemv_layout(NT, b.gs_max);

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(row_blocks, ks, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = L.total;
  cfg.stream = stream;
  cudaLaunchAttribute attrs[2];
  int na = 0;
  if (ks > 1) {
    attrs[na].id = cudaLaunchAttributeClusterDimension;
    attrs[na].val.clusterDim.x = 1;
    attrs[na].val.clusterDim.y = ks;
    attrs[na].val.clusterDim.z = 1;
    ++na;
  }
  if (pdl) {
    attrs[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attrs;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kern, b, static_cast<int>(pdl && static_w), err);
}

}  // namespace

// Adds one linear (one chunk of at most 16 tokens) to a batch.
cudaError_t gemv_batch_add(GemvBatch& b, const void* x, const int32_t* qw, const uint16_t* sc,
                           const uint16_t* z, int N, int K, void* y) {
  const int i = b.count;
  if (encode_2d(&b.tw[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, qw, static_cast<uint64_t>(K) / 2, N,
                static_cast<uint64_t>(K) / 2, 64, kRows, CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (encode_2d(&b.tx[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, K, b.M,
                static_cast<uint64_t>(K) * 2, 64, b.M <= 8 ? 8 : 16,
                CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  b.xp[i] = static_cast<const __nv_bfloat16*>(x);
  b.scales[i] = sc;
  b.zeros[i] = z;
  b.y[i] = static_cast<__nv_bfloat16*>(y);
  b.N[i] = N;
  b.K[i] = K;
  b.cta_start[i + 1] = b.cta_start[i] + (N + kRows - 1) / kRows;
  b.count = i + 1;
  return cudaSuccess;
}

// All items share M (<= 16 tokens) and symmetry.
cudaError_t launch_gemv_batch(GemvBatch& b, bool symmetric, bool pdl, bool static_w,
                              cudaStream_t stream, int num_sms, unsigned* err) {
  if (b.M <= 8)
    return symmetric ? launch_gemv_batch_t<1, true>(b, pdl, static_w, stream, num_sms, err)
                     : launch_gemv_batch_t<1, false>(b, pdl, static_w, stream, num_sms, err);
  return symmetric ? launch_gemv_batch_t<2, true>(b, pdl, static_w, stream, num_sms, err)
                   : launch_gemv_batch_t<2, false>(b, pdl, static_w, stream, num_sms, err);
}

cudaError_t launch_gemv(const void* x, int M, const int32_t* qw, const uint16_t* sc,
                        const uint16_t* z, int N, int K, void* y, bool pdl, bool static_w,
                        cudaStream_t stream, int num_sms, unsigned* err) {
  // M <= 64 in chunks of up to 16 tokens (two n-tiles of 8).
  for (int m0 = 0; m0 < M; m0 += 16) {
    GemvBatch b;
    b.count = 0;
    b.cta_start[0] = 0;
    b.M = (M - m0) < 16 ? (M - m0) : 16;
    const void* xc = static_cast<const __nv_bfloat16*>(x) + static_cast<size_t>(m0) * K;
    void* yc = static_cast<__nv_bfloat16*>(y) + static_cast<size_t>(m0) * N;
    cudaError_t e = gemv_batch_add(b, xc, qw, sc, z, N, K, yc);
    if (e == cudaSuccess) e = launch_gemv_batch(b, z == nullptr, pdl, static_w, stream, num_sms, err);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace w4
