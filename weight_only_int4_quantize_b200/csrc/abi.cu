// extern "C" entry points of libw4 (declared in include/w4.h): host-side
// argument validation, path selection and workspace layout.  Nothing is
// launched unless every check passes; the library allocates nothing.
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <vector>

#include "w4.h"
#include "w4_common.cuh"
#include "w4_kernels.h"

namespace w4 {

// The device error word (one instance per device that loads the library).
__device__ unsigned int g_w4_device_error;

namespace {

constexpr unsigned kKernelIdSelftest = 7;

__global__ void selftest_wait_kernel(unsigned long long limit_ns, unsigned* err) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // Nobody arrives on this barrier: the bounded wait must expire and report.
  if (threadIdx.x == 0) {
    mbar_wait(smem_u32(&bar), 0, &abort_flag, err, kKernelIdSelftest, limit_ns);
  }
  __syncthreads();
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Description of the last W4_ERR_CUDA of this host thread.
thread_local char g_last_error[256] = "";

w4_status cuda_status(cudaError_t e, const char* step = "launch") {
  if (e == cudaSuccess) return W4_OK;
  snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%s)", step, cudaGetErrorName(e),
           cudaGetErrorString(e));
  return W4_ERR_CUDA;
}

w4_status device_info(int* num_sms, unsigned** err_ptr) {
  static int sms[64] = {};
  static unsigned* errp[64] = {};
  int dev = 0;
  cudaError_t ge = cudaGetDevice(&dev);
  if (ge != cudaSuccess) return cuda_status(ge, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return W4_ERR_UNSUPPORTED;
  if (sms[dev] == 0) {
    int n = 0;
    cudaError_t e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_status(e, "SM count");
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_w4_device_error);
    if (e != cudaSuccess) return cuda_status(e, "error word address");
    errp[dev] = static_cast<unsigned*>(p);
    sms[dev] = n;
  }
  *num_sms = sms[dev];
  if (err_ptr) *err_ptr = errp[dev];
  return W4_OK;
}

bool valid_k(int64_t K) { return K >= 128 && K % 128 == 0 && K <= (int64_t{1} << 30); }

size_t round256(size_t b) { return (b + 255) & ~size_t{255}; }

// Workspace of awq_score_grid: every region 256-byte aligned.  xpart, wpart:
// partial column maxima of |x| and |w|; fe: the operand exponents per alpha.
struct AwqWs {
  size_t s, xpart, wpart, fe, a, e, partials, list, rowsum, total;
};

AwqWs awq_layout(int64_t M, int64_t N, int64_t K, int n_alpha, int n_shrink, int n_seg) {
  AwqWs w;
  w.s = 0;
  w.xpart = w.s + round256(sizeof(float) * n_alpha * K);
  w.wpart = w.xpart + round256(sizeof(float) * colmax_chunks(M) * K);
  w.fe = w.wpart + round256(sizeof(float) * colmax_chunks(N) * K);
  w.a = w.fe + round256(sizeof(int) * 2 * n_alpha);
  w.e = w.a + round256(sizeof(uint16_t) * M * K);
  w.partials = w.e + round256(sizeof(uint16_t) * static_cast<size_t>(n_shrink) * N * K);
  const size_t tiles = static_cast<size_t>(sumsq_tiles(static_cast<int>(M), static_cast<int>(N)));
  w.list = w.partials + round256(sizeof(double) * n_alpha * n_shrink * n_seg * tiles);
  w.rowsum = w.list + round256(sizeof(int) * (2 * kExactCap + 1));  // list, count, masks
  w.total = w.rowsum + round256(sizeof(double) * kExactCap *
                                static_cast<size_t>(exact_token_chunks(static_cast<int>(M))) * N);
  return w;
}

// Workspace of awq_clip_search_rows: every region 256-byte aligned.
struct ClipWs {
  size_t ones, xpart, wpart, fe, a, e, partials, flags, list, rows, rowsum, total;
};

ClipWs clip_layout(int64_t M, int64_t N, int64_t K, int n_shrink) {
  ClipWs w;
  w.ones = 0;
  w.xpart = w.ones + round256(sizeof(float) * K);
  w.wpart = w.xpart + round256(sizeof(float) * colmax_chunks(M) * K);
  w.fe = w.wpart + round256(sizeof(float) * colmax_chunks(N) * K);
  w.a = w.fe + round256(sizeof(int) * 2);
  w.e = w.a + round256(sizeof(uint16_t) * M * K);
  w.partials = w.e + round256(sizeof(uint16_t) * static_cast<size_t>(n_shrink) * N * K);
  w.flags = w.partials + round256(sizeof(double) * n_shrink *
                                   static_cast<size_t>(colsumsq_row_tiles(static_cast<int>(M))) * N);
  w.list = w.flags + round256(static_cast<size_t>(n_shrink) * N);
  w.rows = w.list + round256(sizeof(unsigned long long) + sizeof(int) * (2 * kMaxGrid + 1));
  w.rowsum = w.rows + round256(sizeof(int) * static_cast<size_t>(n_shrink) * N);
  w.total = w.rowsum + round256(sizeof(double) * n_shrink *
                                static_cast<size_t>(exact_token_chunks(static_cast<int>(M))) * N);
  return w;
}

// Selections whose fp16 values put candidates within this relative distance
// of the least are decided again in binary64.  Against binary64 values the
// fp16 scores differ by 1.3-2.9e-5 (relative) on tables of 256 or more
// rows of Gaussian or per-channel-scaled heavy-tailed activations (512 to
// 2048 tokens, one linear or the six K = 2048 linears of a Qwen3-1.7B block
// and their sum), and by up to 1.37e-4 where a few outlier input channels
// dominate the error (384 rows x 256 tokens, K = 512, 4 channels x20); a
// single row by up to 6.4e-4.  Half of each tolerance is above those, so two
// candidates whose order the fp16 values could invert are both decided in
// binary64; the GPU tests hold every table to half the tolerance.
constexpr double kGridTieTol = 5e-4;
constexpr double kRowTieTol = 5e-3;

}  // namespace
}  // namespace w4

using namespace w4;

extern "C" {

const char* w4_status_string(w4_status s) {
  switch (s) {
    case W4_OK: return "ok";
    case W4_ERR_INVALID_ARG: return "invalid argument";
    case W4_ERR_SHAPE: return "invalid shape";
    case W4_ERR_ALIGNMENT: return "device pointer not 16-byte aligned";
    case W4_ERR_UNSUPPORTED: return "unsupported configuration";
    case W4_ERR_WORKSPACE: return "workspace missing or too small";
    case W4_ERR_CUDA: return "CUDA runtime error";
    case W4_ERR_DEVICE_TIMEOUT: return "a kernel gave up on a bounded wait";
  }
  return "unknown status";
}

int w4_abi_version(void) { return W4_ABI_VERSION; }

const char* w4_last_error(void) { return g_last_error; }

static w4_status check_quant_item(const void* w_bf16, int64_t N, int64_t K, int symmetric,
                                  const float* awq_s, float shrink, int32_t* qweight,
                                  uint16_t* scales_f16, uint16_t* zeros_f16) {
  if (!w_bf16 || !qweight || !scales_f16) return W4_ERR_INVALID_ARG;
  if ((symmetric != 0) != (zeros_f16 == nullptr)) return W4_ERR_INVALID_ARG;
  if (!(shrink > 0.0f && shrink <= 1.0f)) return W4_ERR_INVALID_ARG;
  if (N < 1 || !valid_k(K) || N > (int64_t{1} << 40) / K) return W4_ERR_SHAPE;
  if (!aligned16(w_bf16) || !aligned16(qweight) || !aligned16(scales_f16) ||
      (zeros_f16 && !aligned16(zeros_f16)) || (awq_s && !aligned16(awq_s)))
    return W4_ERR_ALIGNMENT;
  return W4_OK;
}

w4_status w4_quantize_pack(const void* w_bf16, int64_t N, int64_t K, int group, int symmetric,
                           const float* awq_s, float shrink, int32_t* qweight,
                           uint16_t* scales_f16, uint16_t* zeros_f16, void* stream) {
  if (group != 128 && w_bf16 && qweight && scales_f16) return W4_ERR_UNSUPPORTED;
  w4_status st = check_quant_item(w_bf16, N, K, symmetric, awq_s, shrink, qweight, scales_f16,
                                  zeros_f16);
  if (st != W4_OK) return st;
  if (group != 128) return W4_ERR_UNSUPPORTED;
  int sms = 0;
  unsigned* err = nullptr;
  st = device_info(&sms, &err);
  if (st != W4_OK) return st;
  QuantBatch b;
  b.count = 0;
  b.unit_start[0] = 0;
  quant_batch_add(b, w_bf16, N, K, awq_s, shrink, qweight, scales_f16, zeros_f16);
  return cuda_status(launch_quantize_pack_batch(b, symmetric != 0,
                                                static_cast<cudaStream_t>(stream), sms, err),
                     "quantize+pack launch");
}

w4_status w4_quantize_pack_batched(const w4_quant_item* items, int count, int group,
                                   int symmetric, void* stream) {
  if (!items || count < 1) return W4_ERR_INVALID_ARG;
  if (group != 128) return W4_ERR_UNSUPPORTED;
  for (int i = 0; i < count; ++i) {
    const w4_quant_item& it = items[i];
    const w4_status st = check_quant_item(it.w_bf16, it.N, it.K, symmetric, it.awq_s, it.shrink,
                                          it.qweight, it.scales_f16, it.zeros_f16);
    if (st != W4_OK) return st;
  }
  int sms = 0;
  unsigned* err = nullptr;
  w4_status st = device_info(&sms, &err);
  if (st != W4_OK) return st;
  for (int i0 = 0; i0 < count; i0 += kQuantBatch) {
    QuantBatch b;
    b.count = 0;
    b.unit_start[0] = 0;
    for (int i = i0; i < count && i < i0 + kQuantBatch; ++i) {
      const w4_quant_item& it = items[i];
      quant_batch_add(b, it.w_bf16, it.N, it.K, it.awq_s, it.shrink, it.qweight, it.scales_f16,
                      it.zeros_f16);
    }
    st = cuda_status(launch_quantize_pack_batch(b, symmetric != 0,
                                                static_cast<cudaStream_t>(stream), sms, err),
                     "batched quantize+pack launch");
    if (st != W4_OK) return st;
  }
  return W4_OK;
}

static w4_status check_linear_item(const void* x_bf16, int64_t M, const int32_t* qweight,
                                   const uint16_t* scales_f16, const uint16_t* zeros_f16,
                                   int64_t N, int64_t K, void* y_bf16) {
  if (!x_bf16 || !qweight || !scales_f16 || !y_bf16) return W4_ERR_INVALID_ARG;
  if (M < 1 || N < 1 || !valid_k(K) || M > 0x7FFFFFFF || N > 0x7FFFFFFF) return W4_ERR_SHAPE;
  if (!aligned16(x_bf16) || !aligned16(qweight) || !aligned16(scales_f16) ||
      (zeros_f16 && !aligned16(zeros_f16)) || !aligned16(y_bf16))
    return W4_ERR_ALIGNMENT;
  return W4_OK;
}

static constexpr int64_t kGemvMaxK = 8 * 80 * 128;  // decode kernel: K slice <= 80 groups x 8
static constexpr int64_t kDecodeMaxRows = 32;       // decode kernels up to this M by default

// The persistent streaming decode kernel is chosen for launches that deal
// at least this many 4-warp bundles per SM; smaller launches (a single
// linear, a few short ones) run the per-CTA tensor-map kernel, whose K split
// over a thread-block cluster fills the GPU with few rows.
static constexpr int kStreamMinBundlesPerSm = 2;

static constexpr unsigned kDecodeChoice = W4_LINEAR_DECODE_STREAM | W4_LINEAR_DECODE_TILED;

w4_status w4a16_linear(const void* x_bf16, int64_t M, const int32_t* qweight,
                       const uint16_t* scales_f16, const uint16_t* zeros_f16, int64_t N,
                       int64_t K, int group, void* y_bf16, unsigned flags, void* stream) {
  if (!x_bf16 || !qweight || !scales_f16 || !y_bf16) return W4_ERR_INVALID_ARG;
  const unsigned known = W4_LINEAR_FORCE_GEMV | W4_LINEAR_FORCE_GEMM | W4_LINEAR_PDL |
                         W4_LINEAR_STATIC_WEIGHTS | kDecodeChoice;
  if (flags & ~known) return W4_ERR_INVALID_ARG;
  if ((flags & W4_LINEAR_FORCE_GEMV) && (flags & W4_LINEAR_FORCE_GEMM)) return W4_ERR_INVALID_ARG;
  if ((flags & kDecodeChoice) == kDecodeChoice) return W4_ERR_INVALID_ARG;
  if ((flags & kDecodeChoice) && (flags & W4_LINEAR_FORCE_GEMM)) return W4_ERR_INVALID_ARG;
  if (group != 128) return W4_ERR_UNSUPPORTED;
  w4_status st = check_linear_item(x_bf16, M, qweight, scales_f16, zeros_f16, N, K, y_bf16);
  if (st != W4_OK) return st;
  // The decode kernels keep a CTA's K slice (at most 8 x 80 groups) in a
  // shared scale table; longer K goes to the prefill kernel.
  const bool gemv_ok = K <= kGemvMaxK;
  // Measured on B200: the decode kernels beat the prefill GEMM up to 32
  // tokens on the 27B-scale linears (two 16-token passes still read less
  // than the GEMM's dequantized tiles cost).
  const bool gemv = (flags & (W4_LINEAR_FORCE_GEMV | kDecodeChoice)) ||
                    (M <= kDecodeMaxRows && gemv_ok && !(flags & W4_LINEAR_FORCE_GEMM));
  if (gemv && (M > 64 || !gemv_ok)) return W4_ERR_UNSUPPORTED;
  if ((flags & W4_LINEAR_DECODE_STREAM) && M > 8) return W4_ERR_UNSUPPORTED;
  if (!gemv && (M + 127) / 128 > 65535) return W4_ERR_UNSUPPORTED;
  int sms = 0;
  unsigned* err = nullptr;
  st = device_info(&sms, &err);
  if (st != W4_OK) return st;
  const bool pdl = (flags & W4_LINEAR_PDL) != 0;
  const bool stat = (flags & W4_LINEAR_STATIC_WEIGHTS) != 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (gemv && M <= 8 && !(flags & W4_LINEAR_DECODE_TILED)) {
    StreamBatch b;
    b.count = 0;
    b.unit_start[0] = 0;
    b.M = static_cast<int>(M);
    b.a8 = 0;
    stream_batch_add(b, x_bf16, qweight, scales_f16, zeros_f16, static_cast<int>(N),
                     static_cast<int>(K), y_bf16);
    int bundles = 0;
    st = cuda_status(plan_gemv_stream(b, zeros_f16 == nullptr, sms, &bundles),
                     "decode GEMV plan");
    if (st != W4_OK) return st;
    if ((flags & W4_LINEAR_DECODE_STREAM) || bundles >= kStreamMinBundlesPerSm * sms)
      return cuda_status(launch_gemv_stream(b, zeros_f16 == nullptr, pdl, stat, s, sms),
                         "decode GEMV launch");
  }
  if (gemv)
    return cuda_status(launch_gemv(x_bf16, static_cast<int>(M), qweight, scales_f16, zeros_f16,
                                   static_cast<int>(N), static_cast<int>(K), y_bf16, pdl, stat, s,
                                   sms, err),
                       "decode GEMV launch");
  return cuda_status(launch_prefill_gemm(x_bf16, static_cast<int>(M), qweight, scales_f16,
                                         zeros_f16, static_cast<int>(N), static_cast<int>(K),
                                         y_bf16, pdl, stat, s, err),
                     "prefill tcgen05 GEMM launch");
}

w4_status w4_quantize_act_int8(const void* x_bf16, int64_t M, int64_t K, int8_t* xq_out,
                               int32_t* xsum_out, float* xscale_out, void* stream) {
  if (!x_bf16 || !xq_out || !xsum_out || !xscale_out) return W4_ERR_INVALID_ARG;
  if (M < 1 || M > 0x7FFFFFFF || !valid_k(K)) return W4_ERR_SHAPE;
  if (!aligned16(x_bf16) || !aligned16(xq_out) || !aligned16(xsum_out) || !aligned16(xscale_out))
    return W4_ERR_ALIGNMENT;
  return cuda_status(launch_quantize_act_int8(x_bf16, M, K, xq_out, xsum_out, xscale_out,
                                              static_cast<cudaStream_t>(stream)),
                     "int8 activation quantize launch");
}

static w4_status check_a8_item(const w4a8_item& it, int64_t M) {
  if (!it.xq || !it.xsum || !it.xscale || !it.qweight || !it.scales_f16 || !it.y_bf16)
    return W4_ERR_INVALID_ARG;
  if (M < 1 || it.N < 1 || !valid_k(it.K) || it.N > 0x7FFFFFFF || it.K > kGemvMaxK)
    return W4_ERR_SHAPE;
  if (!aligned16(it.xq) || !aligned16(it.xsum) || !aligned16(it.xscale) ||
      !aligned16(it.qweight) || !aligned16(it.scales_f16) ||
      (it.zeros_f16 && !aligned16(it.zeros_f16)) || !aligned16(it.y_bf16))
    return W4_ERR_ALIGNMENT;
  return W4_OK;
}

w4_status w4a8_linear_batched(const w4a8_item* items, int count, int64_t M, int group,
                              unsigned flags, void* stream) {
  if (!items || count < 1) return W4_ERR_INVALID_ARG;
  if (flags & ~(W4_LINEAR_PDL | W4_LINEAR_STATIC_WEIGHTS)) return W4_ERR_INVALID_ARG;
  if (group != 128) return W4_ERR_UNSUPPORTED;
  if (M > 16) return W4_ERR_UNSUPPORTED;
  const bool sym = items[0].zeros_f16 == nullptr;
  for (int i = 0; i < count; ++i) {
    const w4_status st = check_a8_item(items[i], M);
    if (st != W4_OK) return st;
    if ((items[i].zeros_f16 == nullptr) != sym) return W4_ERR_INVALID_ARG;
  }
  int sms = 0;
  unsigned* err = nullptr;
  w4_status st = device_info(&sms, &err);
  if (st != W4_OK) return st;
  const bool pdl = (flags & W4_LINEAR_PDL) != 0;
  const bool stat = (flags & W4_LINEAR_STATIC_WEIGHTS) != 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  std::vector<int> order(count);
  for (int i = 0; i < count; ++i) order[i] = i;
  std::stable_sort(order.begin(), order.end(),
                   [&](int a, int c) { return items[a].K > items[c].K; });
  // Tokens in chunks of 8 (the kernel's mma columns), linears in launches of
  // up to kStreamBatch, longest K first.
  for (int64_t m0 = 0; m0 < M; m0 += 8) {
    const int mc = static_cast<int>(M - m0 < 8 ? M - m0 : 8);
    for (int i0 = 0; i0 < count;) {
      StreamBatch b;
      b.count = 0;
      b.unit_start[0] = 0;
      b.M = mc;
      b.a8 = 1;
      int j = i0;
      for (; j < count && j < i0 + kStreamBatch; ++j) {
        const w4a8_item& it = items[order[j]];
        if (b.count > 0 && b.unit_start[b.count] + (it.N + 63) / 64 > (int64_t{1} << 30)) break;
        stream_batch_add(b, it.xq + m0 * it.K, it.qweight, it.scales_f16, it.zeros_f16,
                         static_cast<int>(it.N), static_cast<int>(it.K),
                         static_cast<uint16_t*>(it.y_bf16) + m0 * it.N,
                         it.xsum + m0 * (it.K / 128), it.xscale + m0);
      }
      st = cuda_status(launch_gemv_stream(b, sym, pdl, stat, s, sms), "W4A8 decode GEMV launch");
      if (st != W4_OK) return st;
      i0 = j;
    }
  }
  return W4_OK;
}

w4_status w4a8_linear(const int8_t* xq, const int32_t* xsum, const float* xscale, int64_t M,
                      const int32_t* qweight, const uint16_t* scales_f16,
                      const uint16_t* zeros_f16, int64_t N, int64_t K, int group, void* y_bf16,
                      unsigned flags, void* stream) {
  const w4a8_item it{xq, xsum, xscale, qweight, scales_f16, zeros_f16, N, K, y_bf16};
  return w4a8_linear_batched(&it, 1, M, group, flags, stream);
}

// Decodes items idx[0..n) through the per-CTA tensor-map kernel.  Launches
// group the linears by K, largest K first: a launch's shared memory ring is
// sized by its longest K slice, so launches of one K size their CTAs exactly
// (short K fits more CTAs per SM), and no launch ends with a trail of long
// CTAs.  Results do not depend on the grouping.
static w4_status decode_tiled(const w4_linear_item* items, const int* idx, int n, int64_t M,
                              bool sym, bool pdl, bool stat, cudaStream_t s, int sms,
                              unsigned* err) {
  for (int64_t m0 = 0; m0 < M; m0 += 16) {
    const int mc = static_cast<int>(M - m0 < 16 ? M - m0 : 16);
    int64_t k_prev = INT64_MAX;
    for (;;) {
      int64_t kv = 0;  // the largest K below k_prev
      for (int j = 0; j < n; ++j)
        if (items[idx[j]].K < k_prev && items[idx[j]].K > kv) kv = items[idx[j]].K;
      if (kv == 0) break;
      k_prev = kv;
      GemvBatch b;
      b.count = 0;
      b.cta_start[0] = 0;
      b.M = mc;
      for (int j = 0; j <= n; ++j) {
        if (j < n && items[idx[j]].K == kv) {
          const w4_linear_item& it = items[idx[j]];
          const void* xc = static_cast<const uint16_t*>(it.x_bf16) + m0 * it.K;
          void* yc = static_cast<uint16_t*>(it.y_bf16) + m0 * it.N;
          w4_status st = cuda_status(gemv_batch_add(b, xc, it.qweight, it.scales_f16,
                                                    it.zeros_f16, static_cast<int>(it.N),
                                                    static_cast<int>(it.K), yc),
                                     "tensor map");
          if (st != W4_OK) return st;
        }
        if (b.count == kGemvBatch || (j == n && b.count > 0)) {
          w4_status st = cuda_status(launch_gemv_batch(b, sym, pdl, stat, s, sms, err),
                                     "batched decode GEMV launch");
          if (st != W4_OK) return st;
          b.count = 0;
          b.cta_start[0] = 0;
        }
      }
    }
  }
  return W4_OK;
}

w4_status w4_prefill_plan(const int64_t* N, const int64_t* K, int count, int64_t M,
                          const int* resident, int* tile_rows, int* tile_cols, int* k_split) {
  if (!N || !K || !tile_rows || !tile_cols || !k_split) return W4_ERR_INVALID_ARG;
  if (count < 1 || count > 16) return W4_ERR_INVALID_ARG;
  if (M < 1 || M > 0x7FFFFFFF) return W4_ERR_SHAPE;
  int n32[16], k32[16];
  for (int i = 0; i < count; ++i) {
    if (N[i] < 1 || N[i] > 0x7FFFFFFF || !valid_k(K[i])) return W4_ERR_SHAPE;
    n32[i] = static_cast<int>(N[i]);
    k32[i] = static_cast<int>(K[i]);
  }
  int res[kPrefillShapes][kPrefillMaxSplit];
  if (resident) {
    for (int s = 0; s < kPrefillShapes; ++s)
      for (int c = 0; c < kPrefillMaxSplit; ++c) {
        res[s][c] = resident[s * kPrefillMaxSplit + c];
        if (res[s][c] < 1) return W4_ERR_INVALID_ARG;
      }
  } else {
    int sms = 0;
    w4_status st = device_info(&sms, nullptr);
    if (st != W4_OK) return st;
    prefill_resident(sms, nullptr, res);
  }
  const PrefillPlan p = plan_prefill_group(n32, k32, count, static_cast<int>(M), res);
  *tile_rows = p.rows;
  *tile_cols = p.cols;
  *k_split = p.ks;
  return W4_OK;
}

w4_status w4a16_linear_batched(const w4_linear_item* items, int count, int64_t M, int group,
                               unsigned flags, void* stream) {
  if (!items || count < 1) return W4_ERR_INVALID_ARG;
  const unsigned known = W4_LINEAR_PDL | W4_LINEAR_STATIC_WEIGHTS | kDecodeChoice;
  if (flags & ~known) return W4_ERR_INVALID_ARG;
  if ((flags & kDecodeChoice) == kDecodeChoice) return W4_ERR_INVALID_ARG;
  if (group != 128) return W4_ERR_UNSUPPORTED;
  if ((flags & W4_LINEAR_DECODE_STREAM) && M > 8) return W4_ERR_UNSUPPORTED;
  if ((flags & W4_LINEAR_DECODE_TILED) && M > 64) return W4_ERR_UNSUPPORTED;
  const bool sym = items[0].zeros_f16 == nullptr;
  for (int i = 0; i < count; ++i) {
    const w4_linear_item& it = items[i];
    w4_status st = check_linear_item(it.x_bf16, M, it.qweight, it.scales_f16, it.zeros_f16, it.N,
                                     it.K, it.y_bf16);
    if (st != W4_OK) return st;
    if ((it.zeros_f16 == nullptr) != sym) return W4_ERR_INVALID_ARG;
    if ((M <= kDecodeMaxRows || (flags & kDecodeChoice)) && it.K > kGemvMaxK)
      return W4_ERR_UNSUPPORTED;
  }
  int sms = 0;
  unsigned* err = nullptr;
  w4_status st = device_info(&sms, &err);
  if (st != W4_OK) return st;
  const bool pdl = (flags & W4_LINEAR_PDL) != 0;
  const bool stat = (flags & W4_LINEAR_STATIC_WEIGHTS) != 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (M > kDecodeMaxRows && !(flags & kDecodeChoice)) {
    // prefill: grouped tcgen05 launches (up to 16 linears each)
    if ((M + 127) / 128 > 65535) return W4_ERR_UNSUPPORTED;
    std::vector<PrefillItem> pi(count);
    for (int i = 0; i < count; ++i) {
      const w4_linear_item& it = items[i];
      pi[i] = PrefillItem{it.x_bf16, it.qweight, it.scales_f16, it.zeros_f16, it.y_bf16,
                          static_cast<int>(it.N), static_cast<int>(it.K)};
    }
    return cuda_status(launch_prefill_gemm_group(pi.data(), count, static_cast<int>(M), pdl,
                                                 stat, s, err),
                       "grouped prefill tcgen05 GEMM launch");
  }
  std::vector<int> order(count);
  for (int i = 0; i < count; ++i) order[i] = i;
  if (M > 8 || (flags & W4_LINEAR_DECODE_TILED))
    return decode_tiled(items, order.data(), count, M, sym, pdl, stat, s, sms, err);
  // M <= 8: persistent streaming launches of up to kStreamBatch linears,
  // longest K first (the launch deals its units in that order, so the long
  // ones are spread first and the short ones even out the warps' totals);
  // a launch too small to fill the GPU goes to the tensor-map kernel.
  std::stable_sort(order.begin(), order.end(),
                   [&](int a, int c) { return items[a].K > items[c].K; });
  for (int i0 = 0; i0 < count;) {
    StreamBatch b;
    b.count = 0;
    b.unit_start[0] = 0;
    b.M = static_cast<int>(M);
    b.a8 = 0;
    int j = i0;
    // (a launch's bundles are counted in int: at most 2^30 of them)
    for (; j < count && j < i0 + kStreamBatch; ++j) {
      const w4_linear_item& it = items[order[j]];
      if (b.count > 0 && b.unit_start[b.count] + (it.N + 63) / 64 > (int64_t{1} << 30)) break;
      stream_batch_add(b, it.x_bf16, it.qweight, it.scales_f16, it.zeros_f16,
                       static_cast<int>(it.N), static_cast<int>(it.K), it.y_bf16);
    }
    int bundles = 0;
    st = cuda_status(plan_gemv_stream(b, sym, sms, &bundles), "decode GEMV plan");
    if (st != W4_OK) return st;
    if ((flags & W4_LINEAR_DECODE_STREAM) || bundles >= kStreamMinBundlesPerSm * sms)
      st = cuda_status(launch_gemv_stream(b, sym, pdl, stat, s, sms),
                       "batched decode GEMV launch");
    else
      st = decode_tiled(items, order.data() + i0, j - i0, M, sym, pdl, stat, s, sms, err);
    if (st != W4_OK) return st;
    i0 = j;
  }
  return W4_OK;
}

w4_status w4_awq_scales(const void* x_bf16, int64_t M, int64_t K, const float* alphas,
                        int n_alpha, float* s_out, void* stream) {
  if (!x_bf16 || !alphas || !s_out) return W4_ERR_INVALID_ARG;
  if (n_alpha < 1 || n_alpha > kMaxGrid) return W4_ERR_UNSUPPORTED;
  if (M < 1 || K < 1 || M > (int64_t{1} << 31) || K > (int64_t{1} << 31)) return W4_ERR_SHAPE;
  if (!aligned16(x_bf16) || !aligned16(s_out)) return W4_ERR_ALIGNMENT;
  AlphaList al;
  al.n = n_alpha;
  for (int i = 0; i < n_alpha; ++i) {
    if (!std::isfinite(alphas[i])) return W4_ERR_INVALID_ARG;
    al.v[i] = alphas[i];
  }
  int sms = 0;
  w4_status st = device_info(&sms, nullptr);
  if (st != W4_OK) return st;
  return cuda_status(launch_awq_scales(x_bf16, M, K, al, s_out, static_cast<cudaStream_t>(stream)));
}

size_t w4_awq_workspace_bytes(int64_t M, int64_t N, int64_t K, int n_alpha, int n_shrink,
                              int n_seg) {
  if (M < 1 || N < 1 || K < 1 || n_alpha < 1 || n_shrink < 1 || n_seg < 1) return 0;
  return awq_layout(M, N, K, n_alpha, n_shrink, n_seg).total;
}

w4_status awq_score_grid(const void* x_bf16, int64_t M, const void* w_bf16, int64_t N, int64_t K,
                         int group, int symmetric, const float* alphas, int n_alpha,
                         const float* shrinks, int n_shrink, const int64_t* seg_offsets,
                         int n_seg, double* sse_out, int32_t* argmin_out, void* workspace,
                         size_t workspace_bytes, void* stream) {
  if (!x_bf16 || !w_bf16 || !alphas || !shrinks || !sse_out || !argmin_out)
    return W4_ERR_INVALID_ARG;
  if (group != 128) return W4_ERR_UNSUPPORTED;
  if (n_alpha < 1 || n_alpha > kMaxGrid || n_shrink < 1 || n_shrink > kMaxGrid)
    return W4_ERR_UNSUPPORTED;
  if (n_seg < 1 || n_seg > 16) return W4_ERR_UNSUPPORTED;
  if (M < 1 || N < 1 || !valid_k(K) || M > (int64_t{1} << 24) || N > (int64_t{1} << 24))
    return W4_ERR_SHAPE;
  if (seg_offsets == nullptr && n_seg != 1) return W4_ERR_INVALID_ARG;
  int seg[17];
  seg[0] = 0;
  seg[n_seg] = static_cast<int>(N);
  if (seg_offsets) {
    if (seg_offsets[0] != 0 || seg_offsets[n_seg] != N) return W4_ERR_SHAPE;
    for (int i = 1; i < n_seg; ++i) {
      if (seg_offsets[i] <= seg_offsets[i - 1] || seg_offsets[i] % 16 != 0) return W4_ERR_SHAPE;
      seg[i] = static_cast<int>(seg_offsets[i]);
    }
    if (seg_offsets[n_seg] <= seg_offsets[n_seg - 1]) return W4_ERR_SHAPE;
  }
  AlphaList al;
  ShrinkList sl;
  al.n = n_alpha;
  sl.n = n_shrink;
  for (int i = 0; i < n_alpha; ++i) {
    if (!std::isfinite(alphas[i])) return W4_ERR_INVALID_ARG;
    al.v[i] = alphas[i];
  }
  int c1 = 0;
  bool have1 = false;
  for (int j = 0; j < n_shrink; ++j) {
    if (!(shrinks[j] > 0.0f && shrinks[j] <= 1.0f)) return W4_ERR_INVALID_ARG;
    sl.v[j] = shrinks[j];
    if (!have1 && shrinks[j] == 1.0f) {
      c1 = j;
      have1 = true;
    }
  }
  if (!aligned16(x_bf16) || !aligned16(w_bf16) || !aligned16(sse_out) || !aligned16(argmin_out))
    return W4_ERR_ALIGNMENT;
  const AwqWs L = awq_layout(M, N, K, n_alpha, n_shrink, n_seg);
  if (!workspace || workspace_bytes < L.total) return W4_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return W4_ERR_ALIGNMENT;

  int sms = 0;
  unsigned* err = nullptr;
  w4_status st = device_info(&sms, &err);
  if (st != W4_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* s_all = reinterpret_cast<float*>(ws + L.s);
  void* a_buf = ws + L.a;
  void* e_buf = ws + L.e;
  double* partials = reinterpret_cast<double*>(ws + L.partials);
  const int tiles = sumsq_tiles(static_cast<int>(M), static_cast<int>(N));

  float* xpart = reinterpret_cast<float*>(ws + L.xpart);
  float* wpart = reinterpret_cast<float*>(ws + L.wpart);
  int* fe = reinterpret_cast<int*>(ws + L.fe);
  cudaError_t e = launch_awq_scales(x_bf16, M, K, al, s_all, s);
  if (e != cudaSuccess) return cuda_status(e, "awq scales");
  e = launch_colmax_abs(x_bf16, M, K, xpart, s);
  if (e != cudaSuccess) return cuda_status(e, "awq column maxima of x");
  e = launch_colmax_abs(w_bf16, N, K, wpart, s);
  if (e != cudaSuccess) return cuda_status(e, "awq column maxima of w");
  e = launch_awq_exponents(xpart, colmax_chunks(M), wpart, colmax_chunks(N), s_all, n_alpha, K, fe,
                           s);
  if (e != cudaSuccess) return cuda_status(e, "awq operand exponents");
  for (int i = 0; i < n_alpha; ++i) {
    const float* si = s_all + static_cast<size_t>(i) * K;
    e = launch_awq_xs(x_bf16, si, M, K, fe + 2 * i, a_buf, s, sms);
    if (e != cudaSuccess) return cuda_status(e, "awq x/s operand");
    e = launch_awq_err(w_bf16, si, N, K, symmetric != 0, sl, fe + 2 * i + 1, e_buf, s, sms);
    if (e != cudaSuccess) return cuda_status(e, "awq error operand");
    e = launch_sumsq_gemm(a_buf, static_cast<int>(M), e_buf, static_cast<int>(N),
                          static_cast<int>(K), n_shrink,
                          partials + static_cast<size_t>(i) * n_shrink * n_seg * tiles, n_seg, seg,
                          s, err);
    if (e != cudaSuccess) return cuda_status(e, "awq tcgen05 sum-of-squares GEMM");
  }
  e = launch_awq_reduce(partials, n_alpha * n_shrink, n_seg, tiles, n_shrink, fe, sse_out, s);
  if (e != cudaSuccess) return cuda_status(e, "awq reduce");
  SegOffsets so{};
  for (int i = 0; i <= n_seg; ++i) so.off[i] = static_cast<int>(seg[i]);
  // Near ties of any selection: those candidates' SSE again in binary64.
  int* list = reinterpret_cast<int*>(ws + L.list);
  int* count = list + kExactCap;
  uint32_t* masks = reinterpret_cast<uint32_t*>(count + 1);
  double* rowsum = reinterpret_cast<double*>(ws + L.rowsum);
  e = launch_awq_flag(sse_out, n_seg, n_alpha, n_shrink, c1, kGridTieTol, kExactCap, list, count,
                      masks, s);
  if (e != cudaSuccess) return cuda_status(e, "awq near-tie flags");
  e = launch_exact_rowsse(x_bf16, static_cast<int>(M), w_bf16, static_cast<int>(N),
                          static_cast<int>(K), s_all, sl, n_shrink, symmetric != 0, list, count,
                          kExactCap, nullptr, nullptr, masks, so, n_seg, rowsum, s);
  if (e != cudaSuccess) return cuda_status(e, "awq binary64 near-tie scores");
  e = launch_awq_exact_merge(rowsum, static_cast<int>(M), static_cast<int>(N), list, count, masks,
                             kExactCap, n_seg, so, n_alpha * n_shrink, sse_out, s);
  if (e != cudaSuccess) return cuda_status(e, "awq binary64 merge");
  return cuda_status(launch_awq_argmin(sse_out, n_seg, n_alpha, n_shrink, c1, argmin_out, s),
                     "awq argmin");
}

size_t w4_clip_rows_workspace_bytes(int64_t M, int64_t N, int64_t K, int n_shrink) {
  if (M < 1 || N < 1 || K < 1 || n_shrink < 1) return 0;
  return clip_layout(M, N, K, n_shrink).total;
}

w4_status awq_clip_search_rows(const void* x_bf16, int64_t M, const void* w_bf16, int64_t N,
                               int64_t K, int group, int symmetric, const float* awq_s,
                               const float* shrinks, int n_shrink, double* sse_rows_out,
                               int32_t* choice_out, float* shrink_rows_out, void* workspace,
                               size_t workspace_bytes, void* stream) {
  if (!x_bf16 || !w_bf16 || !shrinks || !sse_rows_out || !choice_out) return W4_ERR_INVALID_ARG;
  if (group != 128) return W4_ERR_UNSUPPORTED;
  if (n_shrink < 1 || n_shrink > kMaxGrid) return W4_ERR_UNSUPPORTED;
  if (M < 1 || N < 1 || !valid_k(K) || M > (int64_t{1} << 24) || N > (int64_t{1} << 24))
    return W4_ERR_SHAPE;
  ShrinkList sl;
  sl.n = n_shrink;
  for (int j = 0; j < n_shrink; ++j) {
    if (!(shrinks[j] > 0.0f && shrinks[j] <= 1.0f)) return W4_ERR_INVALID_ARG;
    sl.v[j] = shrinks[j];
  }
  if (!aligned16(x_bf16) || !aligned16(w_bf16) || !aligned16(sse_rows_out) ||
      !aligned16(choice_out) || (awq_s && !aligned16(awq_s)) ||
      (shrink_rows_out && (reinterpret_cast<uintptr_t>(shrink_rows_out) & 3u) != 0))
    return W4_ERR_ALIGNMENT;
  const ClipWs L = clip_layout(M, N, K, n_shrink);
  if (!workspace || workspace_bytes < L.total) return W4_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return W4_ERR_ALIGNMENT;

  int sms = 0;
  unsigned* err = nullptr;
  w4_status st = device_info(&sms, &err);
  if (st != W4_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const float* sv = awq_s;
  cudaError_t e = cudaSuccess;
  if (!sv) {
    float* ones = reinterpret_cast<float*>(ws + L.ones);
    e = launch_fill_ones(ones, K, s);
    if (e != cudaSuccess) return cuda_status(e, "clip search unit scale");
    sv = ones;
  }
  void* a_buf = ws + L.a;
  void* e_buf = ws + L.e;
  double* partials = reinterpret_cast<double*>(ws + L.partials);
  float* xpart = reinterpret_cast<float*>(ws + L.xpart);
  float* wpart = reinterpret_cast<float*>(ws + L.wpart);
  int* fe = reinterpret_cast<int*>(ws + L.fe);
  e = launch_colmax_abs(x_bf16, M, K, xpart, s);
  if (e != cudaSuccess) return cuda_status(e, "clip search column maxima of x");
  e = launch_colmax_abs(w_bf16, N, K, wpart, s);
  if (e != cudaSuccess) return cuda_status(e, "clip search column maxima of w");
  e = launch_awq_exponents(xpart, colmax_chunks(M), wpart, colmax_chunks(N), sv, 1, K, fe, s);
  if (e != cudaSuccess) return cuda_status(e, "clip search operand exponents");
  e = launch_awq_xs(x_bf16, sv, M, K, fe, a_buf, s, sms);
  if (e != cudaSuccess) return cuda_status(e, "clip search x/s operand");
  e = launch_awq_err(w_bf16, sv, N, K, symmetric != 0, sl, fe + 1, e_buf, s, sms);
  if (e != cudaSuccess) return cuda_status(e, "clip search error operand");
  e = launch_colsumsq_gemm(a_buf, static_cast<int>(M), e_buf, static_cast<int>(N),
                           static_cast<int>(K), n_shrink, partials, s, err);
  if (e != cudaSuccess) return cuda_status(e, "clip search tcgen05 column sum-of-squares GEMM");
  e = launch_clip_rows_select(partials, n_shrink, colsumsq_row_tiles(static_cast<int>(M)), N, sl,
                              fe, sse_rows_out, choice_out, shrink_rows_out, s);
  if (e != cudaSuccess) return cuda_status(e, "clip search row selection");
  // Rows with near ties: those ratios' row errors again in binary64.
  uint8_t* flags = ws + L.flags;
  unsigned long long* mask = reinterpret_cast<unsigned long long*>(ws + L.list);
  int* list = reinterpret_cast<int*>(ws + L.list + sizeof(unsigned long long));
  int* count = list + kMaxGrid;
  int* row_counts = count + 1;  // [kMaxGrid]
  return cuda_status(launch_clip_exact(x_bf16, static_cast<int>(M), w_bf16, static_cast<int>(N),
                                       static_cast<int>(K), sv, sl, symmetric != 0, kRowTieTol,
                                       sse_rows_out, choice_out, shrink_rows_out, flags, mask,
                                       list, count, reinterpret_cast<int*>(ws + L.rows),
                                       row_counts, reinterpret_cast<double*>(ws + L.rowsum), s),
                     "clip search binary64 near ties");
}

namespace {

bool valid_block_config(const w4_block_config* c) {
  if (!c) return false;
  if (c->hidden < 128 || c->hidden % 128 != 0 || c->hidden > (1 << 16)) return false;
  if (c->heads < 1 || c->kv_heads < 1 || c->heads % c->kv_heads != 0 || c->heads > 256)
    return false;
  if (c->head_dim != 64 && c->head_dim != 128) return false;
  if ((c->heads * c->head_dim) % 128 != 0) return false;
  if (c->ffn < 128 || c->ffn % 128 != 0 || c->ffn > (1 << 17)) return false;
  return std::isfinite(c->eps) && c->eps > 0.0 && std::isfinite(c->rope_theta) &&
         c->rope_theta > 0.0;
}

// A block's pointers: the seven bf16 linears and the four binary64 gains.
bool block_ptrs(const w4_block_weights* b, BlockLinears* out, bool* aligned) {
  if (!b) return false;
  const void* w[7] = {b->q, b->k, b->v, b->o, b->gate, b->up, b->down};
  const double* g[4] = {b->ln1, b->ln2, b->q_norm, b->k_norm};
  *aligned = true;
  for (int i = 0; i < 7; ++i) {
    if (!w[i]) return false;
    *aligned = *aligned && aligned16(w[i]);
    out->w[i] = w[i];
  }
  for (int i = 0; i < 4; ++i) {
    if (!g[i]) return false;
    *aligned = *aligned && aligned16(g[i]);
  }
  out->norms = BlockNorms{b->ln1, b->ln2, b->q_norm, b->k_norm};
  return true;
}

// Shared checks of the block entry points; fills the internal forms.
w4_status check_block_call(const w4_block_config* cfg, const double* x, int64_t T,
                           const w4_block_weights* block, const w4_block_weights* next,
                           const float* alphas, int n_alpha, const float* shrinks, int n_shrink,
                           void* workspace, size_t workspace_bytes, BlockConfig* c,
                           BlockLinears* bi, BlockLinears* bn) {
  if (!cfg || !x || !block || !alphas || !shrinks) return W4_ERR_INVALID_ARG;
  if (!valid_block_config(cfg)) return W4_ERR_SHAPE;
  if (T < 1 || T > 8192) return W4_ERR_SHAPE;
  if (n_alpha < 1 || n_alpha > kMaxGrid || n_shrink < 1 || n_shrink > kMaxGrid)
    return W4_ERR_UNSUPPORTED;
  for (int i = 0; i < n_alpha; ++i)
    if (!std::isfinite(alphas[i])) return W4_ERR_INVALID_ARG;
  for (int j = 0; j < n_shrink; ++j)
    if (!(shrinks[j] > 0.0f && shrinks[j] <= 1.0f)) return W4_ERR_INVALID_ARG;
  bool al_i = true, al_n = true;
  if (!block_ptrs(block, bi, &al_i)) return W4_ERR_INVALID_ARG;
  if (next && !block_ptrs(next, bn, &al_n)) return W4_ERR_INVALID_ARG;
  if (!al_i || !al_n || !aligned16(x)) return W4_ERR_ALIGNMENT;
  *c = BlockConfig{cfg->hidden, cfg->heads, cfg->kv_heads, cfg->head_dim, cfg->ffn, cfg->eps,
                   cfg->rope_theta};
  if (!workspace || workspace_bytes < block_workspace_bytes(*c, T)) return W4_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return W4_ERR_ALIGNMENT;
  return W4_OK;
}

}  // namespace

size_t w4_block_workspace_bytes(const w4_block_config* cfg, int64_t T) {
  if (!valid_block_config(cfg) || T < 1 || T > 8192) return 0;
  const BlockConfig c{cfg->hidden, cfg->heads, cfg->kv_heads, cfg->head_dim, cfg->ffn, cfg->eps,
                      cfg->rope_theta};
  return block_workspace_bytes(c, T);
}

w4_status awq_block_scoring_losses(const w4_block_config* cfg, const double* x, int64_t T,
                                   const w4_block_weights* block, const w4_block_weights* next,
                                   int group, const float* alphas, int n_alpha,
                                   const float* shrinks, int n_shrink, int symmetric, int only,
                                   double* losses_out, void* workspace, size_t workspace_bytes,
                                   void* stream) {
  if (!losses_out) return W4_ERR_INVALID_ARG;
  if (group < 0 || group > 3) return W4_ERR_INVALID_ARG;
  static const int first[5] = {0, 3, 4, 6, 7};
  if (only != -1 && (only < first[group] || only >= first[group + 1])) return W4_ERR_INVALID_ARG;
  BlockConfig c;
  BlockLinears bi{}, bn{};
  w4_status st = check_block_call(cfg, x, T, block, next, alphas, n_alpha, shrinks, n_shrink,
                                  workspace, workspace_bytes, &c, &bi, &bn);
  if (st != W4_OK) return st;
  if (!aligned16(losses_out)) return W4_ERR_ALIGNMENT;
  int sms = 0;
  unsigned* err = nullptr;
  st = device_info(&sms, &err);
  if (st != W4_OK) return st;
  return cuda_status(block_scoring_losses(&c, x, T, bi, next ? &bn : nullptr, group, alphas,
                                          n_alpha, shrinks, n_shrink, symmetric != 0, only,
                                          losses_out, workspace,
                                          static_cast<cudaStream_t>(stream)),
                     "block-level candidate losses");
}

w4_status awq_block_search(const w4_block_config* cfg, const double* x, int64_t T,
                           const w4_block_weights* block, const w4_block_weights* next,
                           const float* alphas, int n_alpha, const float* shrinks, int n_shrink,
                           int symmetric, int32_t* choice_out, double* losses_out,
                           void* workspace, size_t workspace_bytes, void* stream) {
  if (!choice_out) return W4_ERR_INVALID_ARG;
  BlockConfig c;
  BlockLinears bi{}, bn{};
  w4_status st = check_block_call(cfg, x, T, block, next, alphas, n_alpha, shrinks, n_shrink,
                                  workspace, workspace_bytes, &c, &bi, &bn);
  if (st != W4_OK) return st;
  if (!aligned16(choice_out) || (losses_out && !aligned16(losses_out))) return W4_ERR_ALIGNMENT;
  int sms = 0;
  unsigned* err = nullptr;
  st = device_info(&sms, &err);
  if (st != W4_OK) return st;
  return cuda_status(block_search(&c, x, T, bi, next ? &bn : nullptr, alphas, n_alpha, shrinks,
                                  n_shrink, symmetric != 0, choice_out, losses_out, workspace,
                                  static_cast<cudaStream_t>(stream), err),
                     "block-level search");
}

w4_status w4_quantize_pack_rows(const void* w_bf16, int64_t N, int64_t K, int group,
                                int symmetric, const float* awq_s, const float* shrink_rows,
                                int32_t* qweight, uint16_t* scales_f16, uint16_t* zeros_f16,
                                void* stream) {
  if (!shrink_rows) return W4_ERR_INVALID_ARG;
  if (group != 128 && w_bf16 && qweight && scales_f16) return W4_ERR_UNSUPPORTED;
  w4_status st = check_quant_item(w_bf16, N, K, symmetric, awq_s, 1.0f, qweight, scales_f16,
                                  zeros_f16);
  if (st != W4_OK) return st;
  if (group != 128) return W4_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(shrink_rows) & 3u) != 0) return W4_ERR_ALIGNMENT;
  int sms = 0;
  unsigned* err = nullptr;
  st = device_info(&sms, &err);
  if (st != W4_OK) return st;
  QuantBatch b;
  b.count = 0;
  b.unit_start[0] = 0;
  quant_batch_add(b, w_bf16, N, K, awq_s, 1.0f, qweight, scales_f16, zeros_f16, shrink_rows);
  return cuda_status(launch_quantize_pack_batch(b, symmetric != 0,
                                                static_cast<cudaStream_t>(stream), sms, err),
                     "quantize+pack (per-row shrink) launch");
}

// Variant of awq_score_grid for callers that cannot allocate a workspace:
// the scratch is the library's fixed device array (noalloc.cu).  Nothing here
// allocates; the only CUDA call before the existing entry point is the
// once-per-device address lookup.
w4_status awq_score_grid_static_scratch(const void* x_bf16, int64_t M, const void* w_bf16,
                                        int64_t N, int64_t K, int group, int symmetric,
                                        const float* alphas, int n_alpha, const float* shrinks,
                                        int n_shrink, const int64_t* seg_offsets, int n_seg,
                                        double* sse_out, int32_t* argmin_out, void* stream) {
  // Without a workspace the shared validation checks every argument and
  // launches nothing: any status but W4_ERR_WORKSPACE is an argument error,
  // reported before the scratch is looked up (and reserved).
  const w4_status pre = awq_score_grid(x_bf16, M, w_bf16, N, K, group, symmetric, alphas,
                                       n_alpha, shrinks, n_shrink, seg_offsets, n_seg, sse_out,
                                       argmin_out, nullptr, 0, stream);
  if (pre != W4_ERR_WORKSPACE) return pre;
  const size_t need = w4_awq_workspace_bytes(M, N, K, n_alpha, n_shrink, n_seg);
  if (need > W4_AWQ_STATIC_SCRATCH_BYTES) {
    snprintf(g_last_error, sizeof(g_last_error),
             "awq_score_grid_static_scratch: the problem needs %zu bytes of scratch, the "
             "static scratch holds %zu; use awq_score_grid with a workspace",
             need, static_cast<size_t>(W4_AWQ_STATIC_SCRATCH_BYTES));
    return W4_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  const w4_status st = cuda_status(awq_static_scratch_address(&scratch), "static scratch address");
  if (st != W4_OK) return st;
  return awq_score_grid(x_bf16, M, w_bf16, N, K, group, symmetric, alphas, n_alpha, shrinks,
                        n_shrink, seg_offsets, n_seg, sse_out, argmin_out, scratch,
                        W4_AWQ_STATIC_SCRATCH_BYTES, stream);
}

w4_status w4_device_error(int clear, uint32_t* code_out) {
  unsigned v = 0;
  w4_status st = cuda_status(cudaMemcpyFromSymbol(&v, g_w4_device_error, sizeof(v)),
                             "read device error word");
  if (st != W4_OK) return st;
  if (clear) {
    const unsigned zero = 0;
    st = cuda_status(cudaMemcpyToSymbol(g_w4_device_error, &zero, sizeof(zero)),
                     "clear device error word");
    if (st != W4_OK) return st;
  }
  if (code_out) *code_out = v;
  return v ? W4_ERR_DEVICE_TIMEOUT : W4_OK;
}

w4_status w4_selftest_bounded_wait(uint64_t limit_ns, void* stream) {
  if (limit_ns < 1000000ull || limit_ns > 2000000000ull) return W4_ERR_INVALID_ARG;
  int sms = 0;
  unsigned* err = nullptr;
  w4_status st = device_info(&sms, &err);
  if (st != W4_OK) return st;
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns, err);
  return cuda_status(cudaGetLastError());
}

}  // extern "C"
