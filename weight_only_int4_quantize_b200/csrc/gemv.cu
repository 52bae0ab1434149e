// Decode W4A16 GEMV: y[M, N] = x[M, K] . dequant(Wq)^T for M <= 16 (up to 64
// with W4_LINEAR_FORCE_GEMV).  HBM-bound on the packed weight stream
// (0.53125 B/weight asymmetric, 0.515625 symmetric).
//
// Each warp owns a 16-row weight tile and one K slice.  A lane loads 16
// bytes (32 codes) of two rows per 128-channel group straight into
// registers, dequantizes them to exact bf16 integers (q - zero) with one
// mask/OR and one packed subtract per pair (the canonical nibble order puts
// adjacent channels in nibbles i and i+4), and feeds them as the A fragment
// of mma.m16n8k16 (rows = weights, columns = tokens).  The fp32 group result
// is multiplied by the group scale and accumulated.  The K dimension is
// split over the CTAs of a thread-block cluster; partial sums are reduced in
// rank order through distributed shared memory by the rank-0 CTA (no global
// scratch, deterministic).
//
// Inside one group the mma's 16 reduction slots map to channels as follows:
// lane t (= lane % 4) covers channels 32t..32t+31 of the group, step s
// (0..7) uses channels 32t+4s..32t+4s+3, so the x operand of step s is the
// two consecutive bf16 pairs at that offset and needs no permutation.
#include <cooperative_groups.h>

#include "w4_common.cuh"
#include "w4_kernels.h"

namespace cg = cooperative_groups;

namespace w4 {

namespace {

constexpr int kGemvWarps = 4;
constexpr int kGemvRows = 16 * kGemvWarps;  // weight rows per CTA
constexpr int kGemvUnroll = 4;              // groups of weights in flight

__device__ __forceinline__ uint4 ld_weights(const uint32_t* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ uint4 ld_x(const __nv_bfloat16* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}

// bf16x2 (q_lo - z, q_hi - z) from the nibble pair at bits 0..3 / 16..19 of u.
__device__ __forceinline__ uint32_t dq_pair(uint32_t u, uint32_t zz) {
  const uint32_t b = (u & 0x000F000Fu) | 0x43004300u;  // (128 + q) in each bf16 half
  uint32_t r;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(b), "r"(zz));
  return r;
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// bf16x2 with both halves equal to 128 + z (exact for integer z in 0..15).
__device__ __forceinline__ uint32_t zz_of(float z) {
  const uint32_t h = __bfloat16_as_ushort(__float2bfloat16_rn(128.0f + z));
  return h | (h << 16);
}

template <int NT, bool SYM>
__global__ void __launch_bounds__(kGemvWarps * 32)
    gemv_w4a16_kernel(const __nv_bfloat16* __restrict__ x, const uint32_t* __restrict__ qw,
                      const uint16_t* __restrict__ scales, const uint16_t* __restrict__ zeros,
                      __nv_bfloat16* __restrict__ y, int M, int N, int K, int ksplit,
                      int static_weights) {
  __shared__ float part[NT * 8][kGemvRows];  // [token][row] partial sums of this CTA

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2;
  const int t = lane & 3;
  const int G = K >> 7;
  const int row_blk = blockIdx.x * kGemvRows;
  const int ra = row_blk + warp * 16 + g;  // rows of the A fragment
  const int rb = ra + 8;
  const bool va = ra < N, vb = rb < N;
  const int rank = blockIdx.y;
  const int g_per = (G + ksplit - 1) / ksplit;
  const int g_begin = min(G, rank * g_per);
  const int g_end = min(G, g_begin + g_per);
  const size_t row_words = static_cast<size_t>(K) >> 3;
  const uint32_t* qa = qw + static_cast<size_t>(va ? ra : 0) * row_words + 4 * t;
  const uint32_t* qb = qw + static_cast<size_t>(vb ? rb : 0) * row_words + 4 * t;

  float acc[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[n][i] = 0.f;

  uint4 wa[kGemvUnroll], wb[kGemvUnroll];
  auto load_chunk = [&](int gr0) {
#pragma unroll
    for (int u = 0; u < kGemvUnroll; ++u) {
      const int gr = gr0 + u;
      wa[u] = make_uint4(0, 0, 0, 0);
      wb[u] = make_uint4(0, 0, 0, 0);
      if (gr < g_end) {
        if (va) wa[u] = ld_weights(qa + static_cast<size_t>(gr) * 16);
        if (vb) wb[u] = ld_weights(qb + static_cast<size_t>(gr) * 16);
      }
    }
  };

  // With static weights the first chunk streams in before the dependency
  // wait of a programmatic dependent launch; x and y are only touched after.
  if (static_weights) load_chunk(g_begin);
  pdl_wait();
  if (!static_weights) load_chunk(g_begin);

  for (int gr0 = g_begin; gr0 < g_end; gr0 += kGemvUnroll) {
    if (gr0 != g_begin) load_chunk(gr0);
#pragma unroll
    for (int u = 0; u < kGemvUnroll; ++u) {
      const int gr = gr0 + u;
      if (gr >= g_end) break;
      float sa = 0.f, sb = 0.f, za = 8.f, zb = 8.f;
      if (va) {
        sa = __half2float(__ushort_as_half(scales[static_cast<size_t>(ra) * G + gr]));
        if (!SYM) za = __half2float(__ushort_as_half(zeros[static_cast<size_t>(ra) * G + gr]));
      }
      if (vb) {
        sb = __half2float(__ushort_as_half(scales[static_cast<size_t>(rb) * G + gr]));
        if (!SYM) zb = __half2float(__ushort_as_half(zeros[static_cast<size_t>(rb) * G + gr]));
      }
      const uint32_t zza = zz_of(za), zzb = zz_of(zb);
      // x fragments: token 8n + g, channels 32t .. 32t+31 of the group.
      uint4 xv[NT][4];
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        const int m = 8 * n + g;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          xv[n][j] = make_uint4(0, 0, 0, 0);
          if (m < M) xv[n][j] = ld_x(x + static_cast<size_t>(m) * K + gr * 128 + 32 * t + 8 * j);
        }
      }
      const uint32_t va4[4] = {wa[u].x, wa[u].y, wa[u].z, wa[u].w};
      const uint32_t vb4[4] = {wb[u].x, wb[u].y, wb[u].z, wb[u].w};
      float c[NT][4];
#pragma unroll
      for (int n = 0; n < NT; ++n)
#pragma unroll
        for (int i = 0; i < 4; ++i) c[n][i] = 0.f;
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const int w = s >> 1;
        const int sh = 8 * (s & 1);  // pair 2(s&1) -> shift 4*i
        uint32_t a[4];
        a[0] = dq_pair(va4[w] >> sh, zza);
        a[1] = dq_pair(vb4[w] >> sh, zzb);
        a[2] = dq_pair(va4[w] >> (sh + 4), zza);
        a[3] = dq_pair(vb4[w] >> (sh + 4), zzb);
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          const uint4 xx = xv[n][w];
          const uint32_t b0 = (s & 1) ? xx.z : xx.x;
          const uint32_t b1 = (s & 1) ? xx.w : xx.y;
          mma_bf16_16816(c[n], a, b0, b1);
        }
      }
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        acc[n][0] = fmaf(sa, c[n][0], acc[n][0]);
        acc[n][1] = fmaf(sa, c[n][1], acc[n][1]);
        acc[n][2] = fmaf(sb, c[n][2], acc[n][2]);
        acc[n][3] = fmaf(sb, c[n][3], acc[n][3]);
      }
    }
  }

  // Let the next kernel on the stream begin its prologue.
  pdl_launch_dependents();

  // Stage this CTA's partial sums: token 8n + 2t + {0,1}, rows ra / rb.
  const int lr = warp * 16 + g;
#pragma unroll
  for (int n = 0; n < NT; ++n) {
    part[8 * n + 2 * t][lr] = acc[n][0];
    part[8 * n + 2 * t + 1][lr] = acc[n][1];
    part[8 * n + 2 * t][lr + 8] = acc[n][2];
    part[8 * n + 2 * t + 1][lr + 8] = acc[n][3];
  }

  if (ksplit > 1) {
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    if (rank == 0) {
      for (int e = threadIdx.x; e < NT * 8 * kGemvRows; e += kGemvWarps * 32) {
        const int m = e / kGemvRows;
        const int r = e % kGemvRows;
        float sum = 0.f;
        for (int q = 0; q < ksplit; ++q) {
          const float* rp = cluster.map_shared_rank(&part[0][0], q);
          sum += rp[m * kGemvRows + r];
        }
        const int n_out = row_blk + r;
        if (m < M && n_out < N) y[static_cast<size_t>(m) * N + n_out] = __float2bfloat16_rn(sum);
      }
    }
    cluster.sync();  // peers keep their shared memory alive until rank 0 is done
  } else {
    __syncthreads();
    for (int e = threadIdx.x; e < NT * 8 * kGemvRows; e += kGemvWarps * 32) {
      const int m = e / kGemvRows;
      const int r = e % kGemvRows;
      const int n_out = row_blk + r;
      if (m < M && n_out < N)
        y[static_cast<size_t>(m) * N + n_out] = __float2bfloat16_rn(part[m][r]);
    }
  }
}

template <int NT, bool SYM>
cudaError_t launch_gemv_t(const void* x, int M, const int32_t* qw, const uint16_t* sc,
                          const uint16_t* z, int N, int K, void* y, bool pdl, bool static_w,
                          cudaStream_t stream, int num_sms) {
  const int G = K / 128;
  const int row_blocks = (N + kGemvRows - 1) / kGemvRows;
  int ks = 1;
  while (ks < 8 && row_blocks * ks < 2 * num_sms && G / (ks * 2) >= 2) ks *= 2;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(row_blocks, ks, 1);
  cfg.blockDim = dim3(kGemvWarps * 32, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attrs[2];
  int na = 0;
  attrs[na].id = cudaLaunchAttributeClusterDimension;
  attrs[na].val.clusterDim.x = 1;
  attrs[na].val.clusterDim.y = ks;
  attrs[na].val.clusterDim.z = 1;
  ++na;
  if (pdl) {
    attrs[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attrs[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attrs;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, gemv_w4a16_kernel<NT, SYM>,
                            static_cast<const __nv_bfloat16*>(x),
                            reinterpret_cast<const uint32_t*>(qw), sc, z,
                            static_cast<__nv_bfloat16*>(y), M, N, K, ks,
                            static_cast<int>(pdl && static_w));
}

}  // namespace

cudaError_t launch_gemv(const void* x, int M, const int32_t* qw, const uint16_t* sc,
                        const uint16_t* z, int N, int K, void* y, bool pdl, bool static_w,
                        cudaStream_t stream, int num_sms) {
  const bool sym = (z == nullptr);
  // M <= 64 in chunks of up to 16 tokens (two n-tiles of 8).
  for (int m0 = 0; m0 < M; m0 += 16) {
    const int mc = (M - m0) < 16 ? (M - m0) : 16;
    const void* xc = static_cast<const __nv_bfloat16*>(x) + static_cast<size_t>(m0) * K;
    void* yc = static_cast<__nv_bfloat16*>(y) + static_cast<size_t>(m0) * N;
    cudaError_t e;
    if (mc <= 8) {
      e = sym ? launch_gemv_t<1, true>(xc, mc, qw, sc, z, N, K, yc, pdl, static_w, stream, num_sms)
              : launch_gemv_t<1, false>(xc, mc, qw, sc, z, N, K, yc, pdl, static_w, stream, num_sms);
    } else {
      e = sym ? launch_gemv_t<2, true>(xc, mc, qw, sc, z, N, K, yc, pdl, static_w, stream, num_sms)
              : launch_gemv_t<2, false>(xc, mc, qw, sc, z, N, K, yc, pdl, static_w, stream, num_sms);
    }
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace w4
