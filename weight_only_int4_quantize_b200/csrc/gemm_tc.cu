// tcgen05 GEMM core for sm_100a: D[M, N] = A[M, K] . B[N, K]^T with both
// operands K-major in 128-byte-swizzled shared memory and the fp32
// accumulator in tensor memory.  One CTA computes a tile of 128 or 256 rows
// by 128 or 256 columns.
//
// Warp roles (10 warps):
//   warp 0      TMA producer (A tiles; also B tiles when B comes from TMA)
//   warp 1      TMEM allocation and the single-thread MMA issuer
//   warps 2..9  B producers when B is a packed int4 weight: they stream the
//               codes and scales from global memory, dequantize to bf16 in
//               registers and write the swizzled tile; afterwards all eight
//               run the epilogue (tcgen05.ld -> bf16 store, or sum of squares)
//
// Used by
//   - the W4A16 prefill linear: A = x (bf16, TMA), B = dequant(Wq) (bf16),
//     epilogue stores y in bf16;
//   - AWQ candidate scoring: A = x / s (fp16, TMA), B = W s - w_hat (fp16,
//     TMA, one candidate per grid z), epilogue writes per-tile sums of y^2
//     in binary64 (deterministic order);
//   - the per-output-channel clipping search: the same operands, epilogue
//     writes per-column (output channel) sums of y^2 over the tile's rows in
//     binary64 (deterministic order).
//
// Every mbarrier wait is bounded (w4_common.cuh); a CTA that gives up sets
// the device error word, drains its own TMA loads and MMAs, frees its TMEM
// and returns.  Every TMA load feeds only its own CTA.
#include <cooperative_groups.h>
#include <cudaTypedefs.h>

#include <cmath>

#include "w4_common.cuh"
#include "w4_kernels.h"

namespace w4 {

namespace cg = cooperative_groups;

namespace {

constexpr int BM = 128;   // rows of one UMMA (and of a CTA tile with MT = 1)
constexpr int BN = 256;   // widest B tile (the sum-of-squares GEMM always uses it)
constexpr int BK = 64;
constexpr int kThreads = 320;
constexpr int kProducerWarps = 8;
constexpr int kLoadAhead = 4;  // stages of packed codes in flight per producer thread

// A CTA tile is MT x 128 rows by NB (128 or 256) columns: MT UMMAs per k-step
// share one B tile, so with MT = 2 each dequantized weight feeds twice the
// flops, and NB = 128 halves a CTA's dequantization for grids that would
// otherwise leave SMs idle.  Accumulators: MT x NB fp32 TMEM columns.
template <int MT, int NB>
struct Tile {
  static constexpr uint32_t kTileABytes = MT * BM * BK * 2;  // 16 or 32 KB
  static constexpr uint32_t kTileBBytes = NB * BK * 2;       // 16 or 32 KB
  static constexpr int kStages =
      static_cast<int>((196u * 1024u) / (kTileABytes + kTileBBytes)) > 6
          ? 6
          : static_cast<int>((196u * 1024u) / (kTileABytes + kTileBBytes));
  static constexpr uint32_t kTmemCols = MT * NB;
};

enum : int { kBDequant = 0, kBTma = 1 };
enum : int { kEpiStoreBf16 = 0, kEpiSumSquares = 1, kEpiColSumSquares = 2, kEpiAddF64 = 3 };

constexpr unsigned kKernelIdGemm = 2;

template <int MT, int NB>
struct SmemLayout {
  static constexpr int kStages = Tile<MT, NB>::kStages;
  // offsets from a 1024-byte aligned base
  static constexpr uint32_t a = 0;
  static constexpr uint32_t b = a + kStages * Tile<MT, NB>::kTileABytes;
  static constexpr uint32_t bars = b + kStages * Tile<MT, NB>::kTileBBytes;
  // full_a[S], full_b[S], empty[S], acc_full, done
  static constexpr uint32_t misc = bars + (3 * kStages + 2) * 8;
  // + chunk sums (sum of squares) or per-column sums of the four TMEM lane
  // quarters (column sums of squares): 4 x 256 doubles.
  static constexpr uint32_t total = misc + 64 + 4 * 256 * 8;
  static constexpr size_t bytes = total + 1024;
};

struct SumSqArgs {
  double* partials;     // [n_cand][n_seg][tiles]; column sums: [n_cand][m_tiles][N]
  int n_seg;
  int seg_off[17];      // column (N) boundaries, multiples of 16 inside
  int tiles;            // m_tiles * n_tiles
  // Binary64 accumulate epilogue: out = r1 (+ r2) + 2^-(*ea + *eb) * acc,
  // row pitch ldc.
  double* out;
  const double* r1;
  const double* r2;
  const int* ea;
  const int* eb;
  int ldc;
};

// A prefill launch decodes a group of linears that share the token count:
// CTA tiles of linear i are [tile_start[i], tile_start[i + 1]) of the 1-D
// grid, n-tile fastest (consecutive CTAs share their x tile).
constexpr int kGemmGroup = 16;
struct GemmGroup {
  CUtensorMap ta[kGemmGroup];  // x of each linear, bf16 [M, K], box 64 x (MT x 128)
  const uint32_t* qw[kGemmGroup];
  const uint16_t* scales[kGemmGroup];
  const uint16_t* zeros[kGemmGroup];
  __nv_bfloat16* y[kGemmGroup];
  int N[kGemmGroup];
  int K[kGemmGroup];
  int tile_start[kGemmGroup + 1];
  int count;
};

__device__ __forceinline__ void tma_load_3d(uint32_t smem_dst, const CUtensorMap* map, int c0,
                                            int c1, int c2, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
      : "memory");
}

__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t bf16x2_fma(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t r;
  asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}
__device__ __forceinline__ uint32_t bf16_pair(float v) {
  const uint32_t h = __bfloat16_as_ushort(__float2bfloat16_rn(v));
  return h | (h << 16);
}

// Group constants for the exact bf16 dequantization of one row's group:
// scale = hi + lo with hi = bf16(scale) and lo = scale - hi (exact in bf16:
// the fp16 scale has 11 significant bits).  Then for t = q - z (exact):
// fma(t, hi, t*lo) rounds t*scale once, i.e. equals bf16_rn((q - z)*scale).
struct DqConst {
  uint32_t zz;  // (128 + z) in both halves
  uint32_t hi;
  uint32_t lo;
};

__device__ __forceinline__ DqConst dq_const(float sc, float z) {
  DqConst c;
  const float hi = __bfloat162float(__float2bfloat16_rn(sc));
  c.hi = bf16_pair(hi);
  c.lo = bf16_pair(sc - hi);
  c.zz = bf16_pair(128.0f + z);
  return c;
}

// One packed word (8 codes, nibble order 0,2,4,6,1,3,5,7) -> 8 bf16 in
// channel order (16 bytes).
__device__ __forceinline__ uint4 dq_word(uint32_t v, const DqConst& c) {
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t b = ((v >> (4 * i)) & 0x000F000Fu) | 0x43004300u;
    const uint32_t t = bf16x2_sub(b, c.zz);
    o[i] = bf16x2_fma(t, c.hi, bf16x2_mul(t, c.lo));
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}

template <int BSRC, int EPI, bool SYM, int MT, int NB>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_a,    // kBTma only
                   const __grid_constant__ CUtensorMap tmap_b,    // kBTma only
                   const __grid_constant__ GemmGroup grp,         // kBDequant only
                   const __grid_constant__ SumSqArgs ss,          // sum-of-squares epilogues
                   int M, int N_arg, int K_arg, int pdl_static, unsigned* err) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* base_ptr = smem_raw + (base - raw_addr);

  using SL = SmemLayout<MT, NB>;
  constexpr int kStages = SL::kStages;
  constexpr uint32_t kTileABytes = Tile<MT, NB>::kTileABytes;
  constexpr uint32_t kTileBBytes = Tile<MT, NB>::kTileBBytes;
  constexpr uint32_t kTmemCols = Tile<MT, NB>::kTmemCols;
  const uint32_t sA = base + SL::a;
  const uint32_t sB = base + SL::b;
  const uint32_t bar0 = base + SL::bars;
  auto full_a = [&](int s) { return bar0 + 8u * s; };
  auto full_b = [&](int s) { return bar0 + 8u * (kStages + s); };
  auto empty = [&](int s) { return bar0 + 8u * (2 * kStages + s); };
  const uint32_t acc_full = bar0 + 8u * (3 * kStages);
  const uint32_t done_bar = acc_full + 8u;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base_ptr + SL::misc);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + SL::misc + 8);
  double* chunk_sums = reinterpret_cast<double*>(base_ptr + SL::misc + 64);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // This CTA's operands: the scoring GEMMs take one A and a candidate-indexed
  // B; a prefill CTA finds its linear in the group and its tile in it.
  const CUtensorMap* ta = &tmap_a;
  const uint32_t* __restrict__ qw = nullptr;
  const uint16_t* __restrict__ scales = nullptr;
  const uint16_t* __restrict__ zeros = nullptr;
  __nv_bfloat16* __restrict__ y = nullptr;
  int N = N_arg, K = K_arg;
  int tile_n = blockIdx.x, tile_m = blockIdx.y;
  // Split K over a thread-block cluster (prefill launches whose plan splits K):
  // CTA `rank` of the cluster takes its share of the k-blocks, and the
  // partial accumulators are added through distributed shared memory.
  int ks = 1, rank = 0;
  if constexpr (BSRC == kBDequant) {
    asm("mov.u32 %0, %%cluster_nctarank;" : "=r"(ks));
    asm("mov.u32 %0, %%cluster_ctarank;" : "=r"(rank));
  }
  if constexpr (BSRC == kBDequant) {
    const int cta_tile = static_cast<int>(blockIdx.x) / ks;
    int lo = 0, hi = grp.count - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (grp.tile_start[mid] <= cta_tile) lo = mid; else hi = mid - 1;
    }
    ta = &grp.ta[lo];
    qw = grp.qw[lo];
    scales = grp.scales[lo];
    zeros = grp.zeros[lo];
    y = grp.y[lo];
    N = grp.N[lo];
    K = grp.K[lo];
    const int local = cta_tile - grp.tile_start[lo];
    const int n_tiles = (N + NB - 1) / NB;
    tile_n = local % n_tiles;
    tile_m = local / n_tiles;
  }
  const int n0 = tile_n * NB;
  const int m0 = tile_m * (MT * BM);
  const int cand = blockIdx.z;
  // This CTA's k-blocks: [kb_begin, kb_begin + num_kb); every loop below runs
  // over local indices (stages and phases count from the first local block).
  const int kb_begin = rank * (K / BK) / ks;
  const int num_kb = (rank + 1) * (K / BK) / ks - kb_begin;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_a(s), 1);
      mbar_init(full_b(s), BSRC == kBDequant ? kProducerWarps : 1);
      mbar_init(empty(s), 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(ta);
    if (BSRC == kBTma) tma_prefetch_desc(&tmap_b);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA --
    if (lane == 0) {
      pdl_wait();
      int kb_stop = 0;  // loads for k-blocks [0, kb_stop) were issued
      for (int kb = 0; kb < num_kb; ++kb) {
        const int s = kb % kStages;
        const uint32_t ph = (kb / kStages) & 1u;
        if (!mbar_wait(empty(s), ph ^ 1u, abort_flag, err, kKernelIdGemm)) break;
        if (BSRC == kBTma) {
          mbar_arrive_expect_tx(full_a(s), kTileABytes + kTileBBytes);
          tma_load_2d(sA + s * kTileABytes, ta, (kb_begin + kb) * BK, m0, full_a(s));
          tma_load_3d(sB + s * kTileBBytes, &tmap_b, (kb_begin + kb) * BK, n0, cand, full_a(s));
        } else {
          mbar_arrive_expect_tx(full_a(s), kTileABytes);
          tma_load_2d(sA + s * kTileABytes, ta, (kb_begin + kb) * BK, m0, full_a(s));
        }
        kb_stop = kb + 1;
      }
      if (*abort_flag) {
        // Drain this CTA's own loads before leaving: the last issued k-block
        // of each stage is the only one that can still be in flight.
        for (int kb = kb_stop - kStages; kb < kb_stop; ++kb) {
          if (kb < 0) continue;
          volatile int dummy = 0;
          mbar_wait(full_a(kb % kStages), (kb / kStages) & 1u, &dummy, err, kKernelIdGemm,
                    kWaitLimitNs / 4);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA --
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16(BM, NB, EPI == kEpiStoreBf16);
      bool issued = false;
      for (int kb = 0; kb < num_kb; ++kb) {
        const int s = kb % kStages;
        const uint32_t ph = (kb / kStages) & 1u;
        if (!mbar_wait(full_a(s), ph, abort_flag, err, kKernelIdGemm)) break;
        if (BSRC == kBDequant && !mbar_wait(full_b(s), ph, abort_flag, err, kKernelIdGemm)) break;
        tc_fence_after();
        const uint64_t da = sdesc_k_sw128(sA + s * kTileABytes);
        const uint64_t db = sdesc_k_sw128(sB + s * kTileBBytes);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          // +32 bytes along K inside the swizzle atom = +2 in the address
          // field; row block mt of A starts 16 KB (+1024) further.
#pragma unroll
          for (int mt = 0; mt < MT; ++mt)
            umma_f16(tmem_base + static_cast<uint32_t>(NB) * mt, da + 1024ull * mt + 2ull * kk,
                     db + 2ull * kk, idesc, (kb | kk) != 0);
        }
        issued = true;
        umma_commit(empty(s));
      }
      if (!*abort_flag) {
        umma_commit(acc_full);
      } else if (issued) {
        umma_commit(done_bar);  // wait for in-flight MMAs before TMEM is freed
        volatile int dummy = 0;
        mbar_wait(done_bar, 0, &dummy, err, kKernelIdGemm, kWaitLimitNs / 4);
      }
    }
  } else {
    const int pt = threadIdx.x - 64;  // 0..255
    // ------------------------------------------------- B producers ----
    if (BSRC == kBDequant) {
      // Thread pt owns rows r = it*128 + pt/2 (it < NB / 128) and half (pt & 1)
      // of each row's 64-channel stage slice: 4 packed words -> 4 chunks.
      // A register ring keeps kLoadAhead stages of codes (and their group's
      // scale/zero) in flight ahead of the stage being written.
      const int half = pt & 1;
      const int G = K >> 7;
      const size_t row_words = static_cast<size_t>(K) >> 3;
      int rows[2];
      bool valid[2];
      const uint32_t* qrow[2];
      const uint16_t* srow[2];
      const uint16_t* zrow[2];
#pragma unroll
      for (int it = 0; it < NB / 128; ++it) {
        rows[it] = it * 128 + (pt >> 1);
        valid[it] = (n0 + rows[it]) < N;
        const size_t row = static_cast<size_t>(valid[it] ? n0 + rows[it] : 0);
        qrow[it] = qw + row * row_words + 4 * half;
        srow[it] = scales + row * G;
        zrow[it] = SYM ? nullptr : zeros + row * G;
      }
      uint4 ring[kLoadAhead][2];
      uint32_t ring_sz[kLoadAhead][2];
      auto fetch = [&](int kb, uint4 (&q)[2], uint32_t (&sz)[2]) {
#pragma unroll
        for (int it = 0; it < NB / 128; ++it) {
          q[it] = make_uint4(0, 0, 0, 0);
          sz[it] = 0x48000000u;  // scale 0, zero 8
          if (valid[it] && kb < num_kb) {
            const int ka = kb_begin + kb;  // absolute k-block
            q[it] = __ldg(reinterpret_cast<const uint4*>(qrow[it] + ka * 8));
            sz[it] = srow[it][ka >> 1];
            sz[it] |= SYM ? 0x48000000u : (static_cast<uint32_t>(zrow[it][ka >> 1]) << 16);
          }
        }
      };
      if (pdl_static == 0) pdl_wait();
#pragma unroll
      for (int d = 0; d < kLoadAhead; ++d) fetch(d, ring[d], ring_sz[d]);
      bool stop = false;
      for (int kb0 = 0; kb0 < num_kb && !stop; kb0 += kLoadAhead) {
#pragma unroll
        for (int d = 0; d < kLoadAhead; ++d) {
          const int kb = kb0 + d;
          if (kb >= num_kb) break;
          const int s = kb % kStages;
          const uint32_t ph = (kb / kStages) & 1u;
          const uint4 cur[2] = {ring[d][0], ring[d][1]};
          const uint32_t csz[2] = {ring_sz[d][0], ring_sz[d][1]};
          fetch(kb + kLoadAhead, ring[d], ring_sz[d]);
          DqConst dc[2];
#pragma unroll
          for (int it = 0; it < NB / 128; ++it)
            dc[it] = dq_const(__half2float(__ushort_as_half(static_cast<uint16_t>(csz[it] & 0xFFFFu))),
                              __half2float(__ushort_as_half(static_cast<uint16_t>(csz[it] >> 16))));
          if (!mbar_wait(empty(s), ph ^ 1u, abort_flag, err, kKernelIdGemm)) {
            stop = true;
            break;
          }
          const uint32_t tile = sB + s * kTileBBytes;
#pragma unroll
          for (int it = 0; it < NB / 128; ++it) {
            const uint32_t w4[4] = {cur[it].x, cur[it].y, cur[it].z, cur[it].w};
#pragma unroll
            for (int j = 0; j < 4; ++j)
              st_shared_v4(tile + sw128_offset(rows[it], 4 * half + j), dq_word(w4[j], dc[it]));
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(full_b(s));
        }
      }
      if (pdl_static != 0) pdl_wait();
    }

    if (BSRC == kBTma) pdl_wait();

    // --------------------------------------------------------- epilogue --
    const int q = warp & 3;         // TMEM lane quarter of this warp
    const int ch = (warp - 2) >> 2;  // column half: 0 -> 0..127, 1 -> 128..255
    const bool ok = mbar_wait(acc_full, 0, abort_flag, err, kKernelIdGemm);
    tc_fence_after();
    if (ok) {
      if (EPI == kEpiStoreBf16 && ks > 1) {
        // Split K: this CTA's fp32 partial tile into its own shared memory
        // (the stage buffers are idle once the accumulator is complete),
        // rows padded by 4 words so a warp's 16-byte stores hit distinct
        // banks.  The cluster adds the partials below.
        float* part = reinterpret_cast<float*>(base_ptr + SL::a);
        for (int mt = 0; mt < MT; ++mt)
          for (int c = 0; c < NB / 32; ++c) {
            const int row = 128 * mt + 32 * q + lane;
            const int col = (NB / 2) * ch + 16 * c;
            uint32_t r[16];
            tmem_ld_32x32b_x16(tmem_base + (static_cast<uint32_t>(32 * q) << 16) + NB * mt + col,
                               r);
            tmem_ld_wait();
            float4* dst = reinterpret_cast<float4*>(part + row * (NB + 4) + col);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              dst[i] = make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                                   __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
          }
      } else if (EPI == kEpiStoreBf16) {
        for (int mt = 0; mt < MT; ++mt)
        for (int c = 0; c < NB / 32; ++c) {
          const int m = m0 + 128 * mt + 32 * q + lane;
          const int col = (NB / 2) * ch + 16 * c;
          uint32_t r[16];
          tmem_ld_32x32b_x16(tmem_base + (static_cast<uint32_t>(32 * q) << 16) + NB * mt + col, r);
          tmem_ld_wait();
          const int n = n0 + col;
          if (m < M && n < N) {
            __nv_bfloat16* dst = y + static_cast<size_t>(m) * N + n;
            uint32_t p[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const __nv_bfloat162 b2 =
                  __floats2bfloat162_rn(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
              p[i] = *reinterpret_cast<const uint32_t*>(&b2);
            }
            if (n + 16 <= N && (N & 7) == 0) {
              uint4* d4 = reinterpret_cast<uint4*>(dst);
              d4[0] = make_uint4(p[0], p[1], p[2], p[3]);
              d4[1] = make_uint4(p[4], p[5], p[6], p[7]);
            } else {
              for (int i = 0; i < 16 && n + i < N; ++i)
                dst[i] = __float2bfloat16_rn(__uint_as_float(r[i]));
            }
          }
        }
      } else if (EPI == kEpiAddF64) {
        // out = r1 (+ r2) + 2^-(ea + eb) acc in binary64: the operands were
        // scaled by exact powers of two, which the epilogue removes exactly.
        // Each warp stages its 32 rows x NB/2 columns of fp32 accumulators
        // in the (now idle) stage buffers, rows 132 floats apart, then walks
        // the rows with all 32 lanes on one row, so that r1, r2 and the
        // output move as contiguous runs of the row (4 columns a lane).
        static_assert(EPI != kEpiAddF64 || NB == 256, "binary64 epilogue uses 256-column tiles");
        constexpr int kLd = 132;
        float* stg = reinterpret_cast<float*>(base_ptr + SL::a) + (warp - 2) * (32 * kLd);
        const double scale = ldexp(1.0, -(*ss.ea + *ss.eb));
        const double* r1p = ss.r1;
        const double* r2p = ss.r2;
        double* outp = ss.out;
        for (int mt = 0; mt < MT; ++mt) {
          for (int c = 0; c < NB / 32; ++c) {
            uint32_t r[16];
            tmem_ld_32x32b_x16(
                tmem_base + (static_cast<uint32_t>(32 * q) << 16) + NB * mt + 128 * ch + 16 * c, r);
            tmem_ld_wait();
            float4* d4 = reinterpret_cast<float4*>(stg + lane * kLd + 16 * c);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              d4[i] = make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                                  __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
          }
          __syncwarp();
          const int n = n0 + 128 * ch + 4 * lane;  // this lane's 4 columns
          const bool whole = n + 4 <= N && (ss.ldc & 1) == 0;
          for (int rr = 0; rr < 32; ++rr) {
            const int m = m0 + 128 * mt + 32 * q + rr;
            if (m >= M) break;
            const float4 a = *reinterpret_cast<const float4*>(stg + rr * kLd + 4 * lane);
            const float av[4] = {a.x, a.y, a.z, a.w};
            const size_t o = static_cast<size_t>(m) * ss.ldc + n;
            double v[4], w[4] = {0.0, 0.0, 0.0, 0.0};
            if (whole) {
              const double2 p0 = __ldg(reinterpret_cast<const double2*>(r1p + o));
              const double2 p1 = __ldg(reinterpret_cast<const double2*>(r1p + o) + 1);
              v[0] = p0.x; v[1] = p0.y; v[2] = p1.x; v[3] = p1.y;
              if (r2p) {
                const double2 q0 = __ldg(reinterpret_cast<const double2*>(r2p + o));
                const double2 q1 = __ldg(reinterpret_cast<const double2*>(r2p + o) + 1);
                w[0] = q0.x; w[1] = q0.y; w[2] = q1.x; w[3] = q1.y;
              }
            } else {
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                v[i] = n + i < N ? r1p[o + i] : 0.0;
                if (r2p && n + i < N) w[i] = r2p[o + i];
              }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const double base = r2p ? __dadd_rn(v[i], w[i]) : v[i];
              v[i] = __dadd_rn(base, __dmul_rn(scale, static_cast<double>(av[i])));
            }
            if (whole) {
              reinterpret_cast<double2*>(outp + o)[0] = make_double2(v[0], v[1]);
              reinterpret_cast<double2*>(outp + o)[1] = make_double2(v[2], v[3]);
            } else {
#pragma unroll
              for (int i = 0; i < 4; ++i)
                if (n + i < N) outp[o + i] = v[i];
            }
          }
          __syncwarp();  // the staging rows are rewritten for the next 128-row half
        }
      } else if (EPI == kEpiColSumSquares) {
        // Column sums of y^2 over the tile's rows: per 16-column chunk each
        // thread squares its row's 16 values (its row of each 128-row half
        // in turn), a fixed butterfly over the warp's 32 lanes leaves lane
        // pair (2c, 2c+1) with the sum of the chunk's column c, and the four
        // lane quarters are added in order below.
        static_assert(EPI != kEpiColSumSquares || NB == BN, "column sums use 256-column tiles");
        double* colq = chunk_sums;  // [4][256]
        for (int c = 0; c < 8; ++c) {
          const int col = 128 * ch + 16 * c;
          double d[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) d[i] = 0.0;
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            const int m = m0 + 128 * mt + 32 * q + lane;
            uint32_t r[16];
            tmem_ld_32x32b_x16(tmem_base + (static_cast<uint32_t>(32 * q) << 16) + NB * mt + col,
                               r);
            tmem_ld_wait();
            if (m < M) {
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const double v = static_cast<double>(__uint_as_float(r[i]));
                d[i] = fma(v, v, d[i]);
              }
            }
          }
          // Reduce-scatter: at width w the lanes with bit w set keep the upper
          // half of their columns and receive it from the partner lane.
#pragma unroll
          for (int w = 16, nv = 8; w >= 2; w >>= 1, nv >>= 1) {
            const bool up = (lane & w) != 0;
#pragma unroll
            for (int i = 0; i < nv; ++i) {
              const double keep = up ? d[nv + i] : d[i];
              const double send = up ? d[i] : d[nv + i];
              d[i] = keep + __shfl_xor_sync(0xffffffffu, send, w);
            }
          }
          d[0] += __shfl_xor_sync(0xffffffffu, d[0], 1);
          const int cl = ((lane >> 4) & 1) * 8 + ((lane >> 3) & 1) * 4 + ((lane >> 2) & 1) * 2 +
                         ((lane >> 1) & 1);
          if ((lane & 1) == 0) colq[q * 256 + col + cl] = d[0];
        }
      } else {
        // Sum of squares per 16-column chunk: thread -> fixed-order shuffle
        // tree over the 32 rows of this warp -> shared -> fixed order over
        // the 4 warps of this column half -> per-segment sums.
        // With MT = 2 a thread takes its row of each 128-row half in turn
        // (fixed order).
        static_assert(EPI != kEpiSumSquares || NB == BN, "sum of squares uses 256-column tiles");
        for (int c = 0; c < 8; ++c) {
          const int col = 128 * ch + 16 * c;
          double acc = 0.0;
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            const int m = m0 + 128 * mt + 32 * q + lane;
            uint32_t r[16];
            tmem_ld_32x32b_x16(tmem_base + (static_cast<uint32_t>(32 * q) << 16) + NB * mt + col,
                               r);
            tmem_ld_wait();
            if (m < M) {
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const double v = static_cast<double>(__uint_as_float(r[i]));
                if (n0 + col + i < N) acc = fma(v, v, acc);
              }
            }
          }
#pragma unroll
          for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
          if (lane == 0) chunk_sums[(8 * ch + c) * 4 + q] = acc;
        }
      }
    }
    if (EPI == kEpiColSumSquares) {
      asm volatile("bar.sync 1, 256;" ::: "memory");  // the eight epilogue warps
      const int n = n0 + pt;
      if (n < N && !*abort_flag) {
        const double* colq = chunk_sums;
        const double v = ((colq[pt] + colq[256 + pt]) + colq[512 + pt]) + colq[768 + pt];
        ss.partials[(static_cast<size_t>(cand) * gridDim.y + blockIdx.y) * N + n] = v;
      }
    }
    if (EPI == kEpiSumSquares) {
      asm volatile("bar.sync 1, 256;" ::: "memory");  // the eight epilogue warps
      if (pt < 16) {
        const int chunk = pt;  // 16-column chunk of the tile
        const double v = ((chunk_sums[chunk * 4 + 0] + chunk_sums[chunk * 4 + 1]) +
                          chunk_sums[chunk * 4 + 2]) + chunk_sums[chunk * 4 + 3];
        chunk_sums[64 + chunk] = v;
      }
      asm volatile("bar.sync 1, 256;" ::: "memory");
      if (pt < ss.n_seg && !*abort_flag) {
        double sum = 0.0;
        for (int chunk = 0; chunk < 16; ++chunk) {
          const int c0 = n0 + 16 * chunk;
          if (c0 >= ss.seg_off[pt] && c0 < ss.seg_off[pt + 1]) sum += chunk_sums[64 + chunk];
        }
        const int tile = blockIdx.y * gridDim.x + blockIdx.x;
        ss.partials[(static_cast<size_t>(cand) * ss.n_seg + pt) * ss.tiles + tile] = sum;
      }
    }
  }

  if constexpr (BSRC == kBDequant && EPI == kEpiStoreBf16) {
    if (ks > 1) {
      // Every thread of every CTA of the cluster passes both barriers, also
      // after a timeout (the waits above are bounded), so none is left waiting.
      cg::cluster_group cluster = cg::this_cluster();
      cluster.sync();  // all partial tiles written
      if (warp >= 2 && !*abort_flag) {
        // CTA `rank` adds rows [r0, r1) of the tile over the cluster's CTAs
        // in rank order and stores them (consecutive threads: consecutive
        // columns).
        // Four consecutive columns per thread and four such pieces in flight
        // (distributed shared memory loads have a long latency).
        constexpr int kRows = MT * BM;
        constexpr int kN4 = NB / 4;
        const int r0 = rank * kRows / ks, r1 = (rank + 1) * kRows / ks;
        const int total = (r1 - r0) * kN4;
        float* part = reinterpret_cast<float*>(base_ptr + SL::a);
        for (int e0 = threadIdx.x - 64; e0 < total; e0 += 4 * 256) {
          float4 v[4];
          int off[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int e = e0 + 256 * u;
            off[u] = e < total ? (r0 + e / kN4) * (NB + 4) + 4 * (e % kN4) : -1;
            v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
          }
          for (int p = 0; p < ks; ++p) {  // rank order: the sum is deterministic
            const float* peer = cluster.map_shared_rank(part, p);
            float4 t[4];
#pragma unroll
            for (int u = 0; u < 4; ++u)
              if (off[u] >= 0) t[u] = *reinterpret_cast<const float4*>(peer + off[u]);
#pragma unroll
            for (int u = 0; u < 4; ++u)
              if (off[u] >= 0) {
                v[u].x += t[u].x;
                v[u].y += t[u].y;
                v[u].z += t[u].z;
                v[u].w += t[u].w;
              }
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            if (off[u] < 0) continue;
            const int row = off[u] / (NB + 4), col = off[u] % (NB + 4);
            const int m = m0 + row, n = n0 + col;
            if (m >= M || n >= N) continue;
            __nv_bfloat16* dst = y + static_cast<size_t>(m) * N + n;
            const __nv_bfloat162 lo = __floats2bfloat162_rn(v[u].x, v[u].y);
            const __nv_bfloat162 hi = __floats2bfloat162_rn(v[u].z, v[u].w);
            if (n + 4 <= N && (N & 3) == 0) {
              *reinterpret_cast<uint2*>(dst) =
                  make_uint2(*reinterpret_cast<const uint32_t*>(&lo),
                             *reinterpret_cast<const uint32_t*>(&hi));
            } else {
              const float f[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
              for (int i = 0; i < 4 && n + i < N; ++i) dst[i] = __float2bfloat16_rn(f[i]);
            }
          }
        }
      }
      cluster.sync();  // peers keep their partials until every reader is done
    }
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) pdl_launch_dependents();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

CUresult encode_tmap(CUtensorMap* map, CUtensorMapDataType dt, int rank, const uint64_t* dims,
                     const uint64_t* strides_bytes, const uint32_t* box, const void* base) {
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
  uint32_t estr[3] = {1, 1, 1};
  return fn(map, dt, rank, const_cast<void*>(base), dims, strides_bytes, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

// One instantiation per kernel (the cache below must be per kernel, and
// every instantiation of gemm_tc_kernel has the same function type).
// The scoring GEMMs carry no group.
const GemmGroup kNoGroup = {};

// The opt-in shared-memory size is a per-device function attribute; set it
// once per device and kernel instantiation.
template <auto kern, size_t kSmemBytes>
cudaError_t set_smem_attr() {
  static unsigned long long attr_done = 0;  // bit d: device d
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || !(__atomic_load_n(&attr_done, __ATOMIC_ACQUIRE) & (1ull << dev))) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemBytes));
    if (e != cudaSuccess) return e;
    if (dev < 64) __atomic_fetch_or(&attr_done, 1ull << dev, __ATOMIC_RELEASE);
  }
  return cudaSuccess;
}

// CTAs of the kernel that run at once when launched in clusters of ks
// (1 <= ks <= 4): clusters must fit inside one GPC, so for ks > 1 this can be
// fewer than the SM count.  Queried from the runtime once per device and
// cluster size; while `stream` is being captured into a graph nothing is
// queried, and an unknown value is estimated as whole clusters over the SMs.
template <auto kern, size_t kSmemBytes>
int resident_ctas(int ks, int sms, cudaStream_t stream) {
  if (ks <= 1) return sms;  // one CTA per SM (shared memory)
  static int cache[64][5];  // 0: not known yet
  int dev = 0;
  const int guess = (sms / ks) * ks;
  if (cudaGetDevice(&dev) != cudaSuccess || dev >= 64 || ks > 4) return guess;
  const int known = __atomic_load_n(&cache[dev][ks], __ATOMIC_ACQUIRE);
  if (known > 0) return known;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cap) != cudaSuccess || cap != cudaStreamCaptureStatusNone)
    return guess;
  if (set_smem_attr<kern, kSmemBytes>() != cudaSuccess) return guess;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ks, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeClusterDimension;
  attr.val.clusterDim.x = ks;
  attr.val.clusterDim.y = 1;
  attr.val.clusterDim.z = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = 1;
  int clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&clusters, reinterpret_cast<const void*>(kern), &cfg) !=
          cudaSuccess ||
      clusters <= 0) {
    (void)cudaGetLastError();  // not sticky: clear it, keep the estimate
    return guess;
  }
  const int n = clusters * ks < sms ? clusters * ks : sms;
  __atomic_store_n(&cache[dev][ks], n, __ATOMIC_RELEASE);
  return n;
}

template <auto kern, size_t kSmemBytes>
cudaError_t launch_gemm(dim3 grid, bool pdl, cudaStream_t stream, const CUtensorMap& ta,
                        const CUtensorMap& tb, const GemmGroup& grp, const SumSqArgs& ss, int M,
                        int N, int K, int pdl_static, unsigned* err, int cluster = 1) {
  cudaError_t e = set_smem_attr<kern, kSmemBytes>();
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  if (cluster > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = cluster;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kern, ta, tb, grp, ss, M, N, K, pdl_static, err);
}

}  // namespace

void prefill_resident(int sms, cudaStream_t stream,
                      int (&resident)[kPrefillShapes][kPrefillMaxSplit]) {
  for (int ks = 1; ks <= kPrefillMaxSplit; ++ks) {
    int* r = &resident[0][ks - 1];
    r[0 * kPrefillMaxSplit] = resident_ctas<gemm_tc_kernel<kBDequant, kEpiStoreBf16, true, 2, 256>,
                                            SmemLayout<2, 256>::bytes>(ks, sms, stream);
    r[1 * kPrefillMaxSplit] = resident_ctas<gemm_tc_kernel<kBDequant, kEpiStoreBf16, true, 1, 256>,
                                            SmemLayout<1, 256>::bytes>(ks, sms, stream);
    r[2 * kPrefillMaxSplit] = resident_ctas<gemm_tc_kernel<kBDequant, kEpiStoreBf16, true, 2, 128>,
                                            SmemLayout<2, 128>::bytes>(ks, sms, stream);
    r[3 * kPrefillMaxSplit] = resident_ctas<gemm_tc_kernel<kBDequant, kEpiStoreBf16, true, 1, 128>,
                                            SmemLayout<1, 128>::bytes>(ks, sms, stream);
  }
}

// Tile shape (MT x 128 rows by NB columns, one CTA per SM) and K split
// (clusters of ks <= 4 CTAs, each running 1/ks of the k-blocks, the fp32
// partial tiles added through distributed shared memory) from a time model
// fitted to B200 measurements of single and grouped launches (27B- and
// Llama-2-7B-shaped linears, M = 16 ... 4096; rms error 6 %):
//   waves x (a + b x k-blocks per CTA + (ks > 1 ? c : 0)) microseconds,
//   waves = ceil(tiles x ks / CTAs resident at once),
// the group's tiles counted in units of its longest K.  Per k-block the B
// dequantization of NB columns dominates (two 128-row UMMAs share one
// dequantized tile at about the cost of one); c is the partial-tile
// exchange.  A split needs at least 2 k-blocks per CTA and the partial tile
// must fit the stage buffers.  On equal modelled time the earlier shape and
// the smaller split win.
PrefillPlan plan_prefill_group(const int* N, const int* K, int n, int M,
                               const int (&resident)[kPrefillShapes][kPrefillMaxSplit]) {
  struct Shape { int mt, nb; double a, b, c; size_t stage_bytes; };
  const Shape shapes[kPrefillShapes] = {
      {2, 256, 8.9, 0.923, 0.2, SmemLayout<2, 256>::kStages * size_t(Tile<2, 256>::kTileABytes + Tile<2, 256>::kTileBBytes)},
      {1, 256, 2.5, 0.779, 4.5, SmemLayout<1, 256>::kStages * size_t(Tile<1, 256>::kTileABytes + Tile<1, 256>::kTileBBytes)},
      {2, 128, 7.9, 0.495, 0.9, SmemLayout<2, 128>::kStages * size_t(Tile<2, 128>::kTileABytes + Tile<2, 128>::kTileBBytes)},
      {1, 128, 4.7, 0.482, 1.7, SmemLayout<1, 128>::kStages * size_t(Tile<1, 128>::kTileABytes + Tile<1, 128>::kTileBBytes)}};
  int k_max = 0, kb_min = 1 << 30;
  for (int i = 0; i < n; ++i) {
    k_max = K[i] > k_max ? K[i] : k_max;
    kb_min = K[i] / BK < kb_min ? K[i] / BK : kb_min;
  }
  int best = 1, best_ks = 1;
  double best_cost = -1.0;
  for (int si = 0; si < kPrefillShapes; ++si) {
    const Shape sh = shapes[si];
    if (sh.mt == 2 && M < 2 * BM) continue;  // 256-row tiles only when rows fill them
    double eq = 0.0;  // tiles of the longest K
    for (int i = 0; i < n; ++i)
      eq += static_cast<double>((N[i] + sh.nb - 1) / sh.nb) *
            ((M + sh.mt * BM - 1) / (sh.mt * BM)) * K[i] / k_max;
    const size_t part_bytes = static_cast<size_t>(sh.mt) * BM * (sh.nb + 4) * 4;
    for (int ks = 1; ks <= kPrefillMaxSplit; ++ks) {
      if (ks > 1 && (part_bytes > sh.stage_bytes || kb_min < 2 * ks)) break;
      const int res = resident[si][ks - 1] > 0 ? resident[si][ks - 1] : 1;
      const double waves = std::ceil(eq * ks / res - 1e-9);
      const double cost =
          waves * (sh.a + sh.b * (static_cast<double>(k_max) / BK) / ks + (ks > 1 ? sh.c : 0.0));
      if (best_cost < 0.0 || cost < best_cost - 1e-9) {
        best = si;
        best_ks = ks;
        best_cost = cost;
      }
    }
  }
  return PrefillPlan{shapes[best].mt * BM, shapes[best].nb, best_ks};
}

cudaError_t launch_prefill_gemm_group(const PrefillItem* items_in, int count, int M,
                                      bool pdl, bool static_w, cudaStream_t stream,
                                      unsigned* err) {
  if (count < 1) return cudaSuccess;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int resident[kPrefillShapes][kPrefillMaxSplit];
  prefill_resident(sms, stream, resident);
  // Longest K first: the long CTAs start first and the short ones fill in.
  PrefillItem items[kGemmGroup];
  for (int i0 = 0; i0 < count; i0 += kGemmGroup) {
    const int n = count - i0 < kGemmGroup ? count - i0 : kGemmGroup;
    for (int i = 0; i < n; ++i) items[i] = items_in[i0 + i];
    for (int i = 1; i < n; ++i)
      for (int j = i; j > 0 && items[j].K > items[j - 1].K; --j) {
        const PrefillItem t = items[j];
        items[j] = items[j - 1];
        items[j - 1] = t;
      }
    const bool sym = items[0].z == nullptr;
    int Ns[kGemmGroup], Ks[kGemmGroup];
    for (int i = 0; i < n; ++i) {
      Ns[i] = items[i].N;
      Ks[i] = items[i].K;
    }
    const PrefillPlan plan = plan_prefill_group(Ns, Ks, n, M, resident);
    const int mt = plan.rows / BM, nb = plan.cols;
    const int ks = plan.ks;
    const int bm = mt * BM;
    GemmGroup grp;
    grp.count = n;
    grp.tile_start[0] = 0;
    for (int i = 0; i < n; ++i) {
      const PrefillItem& it = items[i];
      const uint64_t dims[2] = {static_cast<uint64_t>(it.K), static_cast<uint64_t>(M)};
      const uint64_t str[1] = {static_cast<uint64_t>(it.K) * 2};
      const uint32_t box[2] = {BK, static_cast<uint32_t>(bm)};
      if (encode_tmap(&grp.ta[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, dims, str, box, it.x) !=
          CUDA_SUCCESS)
        return cudaErrorInvalidValue;
      grp.qw[i] = reinterpret_cast<const uint32_t*>(it.qw);
      grp.scales[i] = it.sc;
      grp.zeros[i] = it.z;
      grp.y[i] = static_cast<__nv_bfloat16*>(it.y);
      grp.N[i] = it.N;
      grp.K[i] = it.K;
      const long tiles = static_cast<long>((it.N + nb - 1) / nb) * ((M + bm - 1) / bm);
      if (grp.tile_start[i] + tiles > 0x7FFFFFFFL) return cudaErrorInvalidValue;
      grp.tile_start[i + 1] = grp.tile_start[i] + static_cast<int>(tiles);
    }
    CUtensorMap none = grp.ta[0];  // unused by the dequantizing variant
    SumSqArgs ss = {};
    if (static_cast<long>(grp.tile_start[n]) * ks > 0x7FFFFFFFL) return cudaErrorInvalidValue;
    dim3 grid(grp.tile_start[n] * ks, 1, 1);
    const int ps = (pdl && static_w) ? 1 : 0;
    cudaError_t e;
#define W4_PREFILL_LAUNCH(MT_, NB_)                                                           \
  (sym ? launch_gemm<gemm_tc_kernel<kBDequant, kEpiStoreBf16, true, MT_, NB_>,                \
                     SmemLayout<MT_, NB_>::bytes>(grid, pdl, stream, none, none, grp, ss, M, 0, \
                                                  0, ps, err, ks)                             \
       : launch_gemm<gemm_tc_kernel<kBDequant, kEpiStoreBf16, false, MT_, NB_>,               \
                     SmemLayout<MT_, NB_>::bytes>(grid, pdl, stream, none, none, grp, ss, M, 0, \
                                                  0, ps, err, ks))
    if (mt == 2 && nb == 256) e = W4_PREFILL_LAUNCH(2, 256);
    else if (mt == 2) e = W4_PREFILL_LAUNCH(2, 128);
    else if (nb == 256) e = W4_PREFILL_LAUNCH(1, 256);
    else e = W4_PREFILL_LAUNCH(1, 128);
#undef W4_PREFILL_LAUNCH
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_prefill_gemm(const void* x, int M, const int32_t* qw, const uint16_t* sc,
                                const uint16_t* z, int N, int K, void* y, bool pdl,
                                bool static_w, cudaStream_t stream, unsigned* err) {
  const PrefillItem it{x, qw, sc, z, y, N, K};
  return launch_prefill_gemm_group(&it, 1, M, pdl, static_w, stream, err);
}

// Row tiles of the sum-of-squares GEMM: 256 rows (two UMMAs per k-step
// sharing each B tile) whenever M fills them.
int sumsq_mt(int M) { return M >= 2 * BM ? 2 : 1; }

cudaError_t launch_sumsq_gemm(const void* a_f16, int M, const void* b_f16, int N, int K,
                              int n_cand, double* partials, int n_seg, const int* seg_off,
                              cudaStream_t stream, unsigned* err) {
  CUtensorMap ta, tb;
  const uint64_t da[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(M)};
  const uint64_t sa[1] = {static_cast<uint64_t>(K) * 2};
  const int mt = sumsq_mt(M);
  const uint32_t ba[2] = {BK, static_cast<uint32_t>(mt * BM)};
  if (encode_tmap(&ta, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, da, sa, ba, a_f16) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const uint64_t db[3] = {static_cast<uint64_t>(K), static_cast<uint64_t>(N),
                          static_cast<uint64_t>(n_cand)};
  const uint64_t sb[2] = {static_cast<uint64_t>(K) * 2, static_cast<uint64_t>(K) * 2 * N};
  const uint32_t bb[3] = {BK, BN, 1};
  if (encode_tmap(&tb, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, db, sb, bb, b_f16) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  SumSqArgs ss = {};
  ss.partials = partials;
  ss.n_seg = n_seg;
  for (int i = 0; i <= n_seg; ++i) ss.seg_off[i] = seg_off[i];
  dim3 grid((N + BN - 1) / BN, (M + mt * BM - 1) / (mt * BM), n_cand);
  ss.tiles = grid.x * grid.y;
  if (mt == 2)
    return launch_gemm<gemm_tc_kernel<kBTma, kEpiSumSquares, false, 2, BN>,
                       SmemLayout<2, BN>::bytes>(grid, false, stream, ta, tb, kNoGroup, ss, M, N,
                                                 K, 0, err);
  return launch_gemm<gemm_tc_kernel<kBTma, kEpiSumSquares, false, 1, BN>, SmemLayout<1, BN>::bytes>(
      grid, false, stream, ta, tb, kNoGroup, ss, M, N, K, 0, err);
}

cudaError_t launch_add_gemm_f16(const void* a_f16, int M, const void* b_f16, int N, int K,
                                double* out, int ldc, const double* r1, const double* r2,
                                const int* ea, const int* eb, cudaStream_t stream,
                                unsigned* err) {
  if (K % BK != 0) return cudaErrorInvalidValue;
  CUtensorMap ta, tb;
  const uint64_t da[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(M)};
  const uint64_t sa[1] = {static_cast<uint64_t>(K) * 2};
  // 256-row tiles share each B tile between two UMMAs, but only when their
  // count still covers the SMs; otherwise 128-row tiles double the CTAs.
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long tiles2 = static_cast<long>((N + BN - 1) / BN) * ((M + 2 * BM - 1) / (2 * BM));
  const int mt = (M >= 2 * BM && tiles2 >= sms) ? 2 : 1;
  const uint32_t ba[2] = {BK, static_cast<uint32_t>(mt * BM)};
  if (encode_tmap(&ta, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, da, sa, ba, a_f16) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const uint64_t db[3] = {static_cast<uint64_t>(K), static_cast<uint64_t>(N), 1};
  const uint64_t sb[2] = {static_cast<uint64_t>(K) * 2, static_cast<uint64_t>(K) * 2 * N};
  const uint32_t bb[3] = {BK, BN, 1};
  if (encode_tmap(&tb, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, db, sb, bb, b_f16) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  SumSqArgs ss = {};
  ss.out = out;
  ss.r1 = r1;
  ss.r2 = r2;
  ss.ea = ea;
  ss.eb = eb;
  ss.ldc = ldc;
  dim3 grid((N + BN - 1) / BN, (M + mt * BM - 1) / (mt * BM), 1);
  if (mt == 2)
    return launch_gemm<gemm_tc_kernel<kBTma, kEpiAddF64, false, 2, BN>, SmemLayout<2, BN>::bytes>(
        grid, false, stream, ta, tb, kNoGroup, ss, M, N, K, 0, err);
  return launch_gemm<gemm_tc_kernel<kBTma, kEpiAddF64, false, 1, BN>, SmemLayout<1, BN>::bytes>(
      grid, false, stream, ta, tb, kNoGroup, ss, M, N, K, 0, err);
}

cudaError_t launch_colsumsq_gemm(const void* a_f16, int M, const void* b_f16, int N, int K,
                                 int n_cand, double* partials, cudaStream_t stream,
                                 unsigned* err) {
  CUtensorMap ta, tb;
  const uint64_t da[2] = {static_cast<uint64_t>(K), static_cast<uint64_t>(M)};
  const uint64_t sa[1] = {static_cast<uint64_t>(K) * 2};
  const int mt = sumsq_mt(M);
  const uint32_t ba[2] = {BK, static_cast<uint32_t>(mt * BM)};
  if (encode_tmap(&ta, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, da, sa, ba, a_f16) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const uint64_t db[3] = {static_cast<uint64_t>(K), static_cast<uint64_t>(N),
                          static_cast<uint64_t>(n_cand)};
  const uint64_t sb[2] = {static_cast<uint64_t>(K) * 2, static_cast<uint64_t>(K) * 2 * N};
  const uint32_t bb[3] = {BK, BN, 1};
  if (encode_tmap(&tb, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, db, sb, bb, b_f16) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  SumSqArgs ss = {};
  ss.partials = partials;
  dim3 grid((N + BN - 1) / BN, (M + mt * BM - 1) / (mt * BM), n_cand);
  ss.tiles = grid.x * grid.y;
  if (mt == 2)
    return launch_gemm<gemm_tc_kernel<kBTma, kEpiColSumSquares, false, 2, BN>,
                       SmemLayout<2, BN>::bytes>(grid, false, stream, ta, tb, kNoGroup, ss, M, N,
                                                 K, 0, err);
  return launch_gemm<gemm_tc_kernel<kBTma, kEpiColSumSquares, false, 1, BN>,
                     SmemLayout<1, BN>::bytes>(grid, false, stream, ta, tb, kNoGroup, ss, M, N,
                                               K, 0, err);
}

int colsumsq_row_tiles(int M) { return (M + sumsq_mt(M) * BM - 1) / (sumsq_mt(M) * BM); }

int sumsq_tiles(int M, int N) {
  return ((N + BN - 1) / BN) * ((M + sumsq_mt(M) * BM - 1) / (sumsq_mt(M) * BM));
}

}  // namespace w4
