// api.cu - the C ABI declared in include/tiled_attention.h: argument checks, TMA descriptors,
// workspace layout and kernel launches.  One translation unit holds every kernel, so the device
// status word below is a single symbol per GPU.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "tiled_attention.h"

#include "attn_fwd_kernels.cuh"
#include "attn_fwd_persistent.cuh"
#include "decode_kernels.cuh"
#include "merge_kernels.cuh"
#include "prepass_kernels.cuh"

namespace {

using namespace tattn;

thread_local char g_last_cuda_error[256] = "";
constexpr int kMaxDevices = 64;

int cuda_fail(cudaError_t e, const char* what) {
  std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s: %s", what, cudaGetErrorString(e));
  return ATTN_ERR_LAUNCH;
}
#define TATTN_CUDA(call)                             \
  do {                                               \
    cudaError_t e_ = (call);                         \
    if (e_ != cudaSuccess) return cuda_fail(e_, #call); \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

int check_shape(int B, int Hq, int Hkv, int N, int d) {
  if (B < 1 || Hq < 1 || Hkv < 1 || N < 1) return ATTN_ERR_ARG;
  if (Hq % Hkv) return ATTN_ERR_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  // kernels index with 32-bit grid coordinates and TMA rows; keep every extent well inside that
  const long long rows = (long long)B * Hq * N;
  if (rows > (1ll << 31) - 1 || (long long)B * Hq > (1 << 30) || N > (1 << 30)) return ATTN_ERR_UNSUPPORTED;
  return ATTN_OK;
}

#include "tma_host.cuh"
#include "decode_launch.cuh"
#include "attn_fwd_launch.cuh"

int check_common(const void* q, const void* k, const void* v, const void* o, const float* lse, int B, int Hq,
                 int Hkv, int N, int d, int causal, float scale, int dtype) {
  if (!q || !k || !v || !o) return ATTN_ERR_ARG;
  if (causal != 0 && causal != 1) return ATTN_ERR_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_ARG;
  if (dtype != ATTN_BF16 && dtype != ATTN_FP16) return ATTN_ERR_ARG;
  int rc = check_shape(B, Hq, Hkv, N, d);
  if (rc) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || (lse && !aligned16(lse)))
    return ATTN_ERR_ALIGN;
  return ATTN_OK;
}

// ----------------------------------------- workspace layout ---------------------------------------
struct WsLayout {
  size_t q8, k8, sq, sk, kmean, bias, scratch, total;
};

size_t scratch_bytes(int B, int Hkv, int N, int d) {
  const size_t T = ((size_t)N + 127) / 128;
  return align256((size_t)B * Hkv * T * d * sizeof(double));
}

WsLayout ws_layout(int B, int Hq, int Hkv, int N, int d) {
  const size_t T = ((size_t)N + 127) / 128;
  WsLayout w{};
  size_t off = 0;
  w.q8 = off;      off += align256((size_t)B * Hq * N * d);
  w.k8 = off;      off += align256((size_t)B * Hkv * N * d);
  w.sq = off;      off += align256((size_t)B * Hq * T * 4);
  w.sk = off;      off += align256((size_t)B * Hkv * T * 4);
  w.kmean = off;   off += align256((size_t)B * Hkv * d * 4);
  w.bias = off;    off += align256((size_t)B * Hq * N * 4);
  w.scratch = off; off += scratch_bytes(B, Hkv, N, d);
  w.total = off;
  return w;
}

template <bool F8>
int launch_quant(const uint16_t* q16, const uint16_t* k16, int B, int Hq, int Hkv, int N, int d, bool fp16,
                 float scale, const float* kmean, int8_t* q8, float* sq, int8_t* k8, float* sk, float* bias,
                 unsigned qblocks, cudaStream_t stream) {
  if (d == 128) {
    if (fp16)
      quant_kernel<128, true, F8><<<qblocks, quant_threads<128>(), 0, stream>>>(q16, k16, B, Hq, Hkv, N, scale, kmean, q8, sq, k8, sk, bias);
    else
      quant_kernel<128, false, F8><<<qblocks, quant_threads<128>(), 0, stream>>>(q16, k16, B, Hq, Hkv, N, scale, kmean, q8, sq, k8, sk, bias);
  } else {
    if (fp16)
      quant_kernel<64, true, F8><<<qblocks, quant_threads<64>(), 0, stream>>>(q16, k16, B, Hq, Hkv, N, scale, kmean, q8, sq, k8, sk, bias);
    else
      quant_kernel<64, false, F8><<<qblocks, quant_threads<64>(), 0, stream>>>(q16, k16, B, Hq, Hkv, N, scale, kmean, q8, sq, k8, sk, bias);
  }
  TATTN_CUDA(cudaGetLastError());
  return ATTN_OK;
}

// Once per device and kernel: allow `bytes` of dynamic shared memory.
template <class Kern>
int allow_dynamic_smem(Kern kern, int bytes, std::atomic<int>* done) {
  int dev = 0;
  TATTN_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_LAUNCH;
  if (done[dev].load(std::memory_order_acquire) != 1) {
    TATTN_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
    done[dev].store(1, std::memory_order_release);
  }
  return ATTN_OK;
}

// The pre-pass: K channel mean (float64 partials, then the final division), then smoothing and
// quantisation of K and quantisation of Q with the lse bias; f8 selects E4M3 codes over INT8.
int launch_prepass(const void* q, const void* k, int B, int Hq, int Hkv, int N, int d, int dtype, float scale,
                   int8_t* q8, float* sq, int8_t* k8, float* sk, float* kmean, float* bias, double* part,
                   cudaStream_t stream, bool f8 = false) {
  const int T = (N + 127) / 128;
  const int BG = B * Hkv;
  const bool fp16 = dtype == ATTN_FP16;
  const auto* k16 = static_cast<const uint16_t*>(k);
  const auto* q16 = static_cast<const uint16_t*>(q);
  {
    const unsigned blocks = (unsigned)((long long)BG * T);
    if (d == 128) {
      if (fp16) kmean_partial_kernel<128, true><<<blocks, 128, 0, stream>>>(k16, N, part);
      else kmean_partial_kernel<128, false><<<blocks, 128, 0, stream>>>(k16, N, part);
    } else {
      if (fp16) kmean_partial_kernel<64, true><<<blocks, 64, 0, stream>>>(k16, N, part);
      else kmean_partial_kernel<64, false><<<blocks, 64, 0, stream>>>(k16, N, part);
    }
    TATTN_CUDA(cudaGetLastError());
  }
  if (d == 128) {
    static std::atomic<int> set128[kMaxDevices];
    int rc = allow_dynamic_smem(kmean_final_kernel<128>, kmean_final_smem<128>(), set128);
    if (rc) return rc;
    kmean_final_kernel<128><<<BG, kFinalThreads, kmean_final_smem<128>(), stream>>>(part, N, kmean);
  } else {
    static std::atomic<int> set64[kMaxDevices];
    int rc = allow_dynamic_smem(kmean_final_kernel<64>, kmean_final_smem<64>(), set64);
    if (rc) return rc;
    kmean_final_kernel<64><<<BG, kFinalThreads, kmean_final_smem<64>(), stream>>>(part, N, kmean);
  }
  TATTN_CUDA(cudaGetLastError());
  const unsigned qblocks = (unsigned)((long long)B * Hkv * T + (long long)B * Hq * T);
  return f8 ? launch_quant<true>(q16, k16, B, Hq, Hkv, N, d, fp16, scale, kmean, q8, sq, k8, sk, bias, qblocks, stream)
            : launch_quant<false>(q16, k16, B, Hq, Hkv, N, d, fp16, scale, kmean, q8, sq, k8, sk, bias, qblocks, stream);
}

int fwd_quantized(const void* q8, const float* sq, const void* k8, const float* sk, const float* bias, const void* v,
                  void* o, float* lse, int B, int Hq, int Hkv, int N, int d, int causal, float scale, int dtype,
                  bool f8, cudaStream_t stream) {
  FwdParams p = make_params(B, Hq, Hkv, N, causal, scale, o, lse);
  p.sq = sq;
  p.sk = sk;
  p.bias = bias;
  return f8 ? launch_fwd<QK_F8>(q8, k8, v, d, dtype, p, stream) : launch_fwd<QK_I8>(q8, k8, v, d, dtype, p, stream);
}

__global__ void exp2_eval_kernel(const float* __restrict__ x, float* __restrict__ y, int n, int use_poly) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (use_poly == 2) {  // packed pairs, as the softmax evaluates them
    if (2 * i + 1 < n) {
      const float2 r = exp2_poly2(make_float2(x[2 * i], x[2 * i + 1]));
      y[2 * i] = r.x;
      y[2 * i + 1] = r.y;
    } else if (2 * i < n) {
      y[2 * i] = exp2_poly2(make_float2(x[2 * i], 0.f)).x;
    }
    return;
  }
  if (i < n) y[i] = use_poly ? exp2_poly(x[i]) : ex2_approx(x[i]);
}

__global__ void wait_forever_probe_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // nothing ever arrives on `bar`: the wait must give up after limit_ns and report it
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, 0x7f, limit_ns);
}

// ------------------------------------------------------------------------------------------------
// Allocation-free pre-pass.  The only device memory attn_quant_smooth_k needs beyond its inputs and
// outputs is the float64 block partials of the K mean; this variant keeps them in a fixed array
// that lives in the library itself, so a caller that cannot allocate device memory still gets the
// same pre-pass.  The array is file-scope and holds up to kStaticScratchBytes; every GPU that loads
// the library holds its own copy until the process exits.  Its host-side name is only a stand-in,
// so its device address is looked up once per device (cudaGetSymbolAddress, with that device
// current) and cached; kernels are given that address.
// ------------------------------------------------------------------------------------------------
constexpr size_t kStaticScratchBytes = size_t(8) << 20;  // 8 MiB = 1 Mi float64 partials
static __device__ __align__(256) double g_static_kmean_scratch[kStaticScratchBytes / sizeof(double)];

std::mutex g_static_scratch_mu;
void* g_static_scratch_addr[kMaxDevices] = {};

int static_scratch_address(double** out) {
  int dev = -1;
  TATTN_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) {
    std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "device ordinal %d out of range", dev);
    return ATTN_ERR_LAUNCH;
  }
  std::lock_guard<std::mutex> lock(g_static_scratch_mu);
  if (g_static_scratch_addr[dev] == nullptr) {
    void* addr = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&addr, g_static_kmean_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static K-mean scratch)");
    g_static_scratch_addr[dev] = addr;
  }
  *out = static_cast<double*>(g_static_scratch_addr[dev]);
  return ATTN_OK;
}

}  // namespace

extern "C" {

size_t attn_workspace_bytes(int B, int Hq, int Hkv, int N, int d, int mode) {
  if (mode != ATTN_MODE_INT8_QK && mode != ATTN_MODE_FP8_QK) return 0;
  if (check_shape(B, Hq, Hkv, N, d)) return 0;
  return ws_layout(B, Hq, Hkv, N, d).total;
}

size_t attn_quant_scratch_bytes(int B, int Hkv, int N, int d) {
  if (B < 1 || Hkv < 1 || N < 1 || (d != 64 && d != 128)) return 0;
  return scratch_bytes(B, Hkv, N, d);
}

int attn_quant_smooth_k(const void* q, const void* k, int B, int Hq, int Hkv, int N, int d, int dtype, float scale,
                        int8_t* q8, float* sq, int8_t* k8, float* sk, float* kmean, float* lse_bias, void* scratch,
                        size_t scratch_bytes_given, void* stream) {
  if (!q || !k || !q8 || !sq || !k8 || !sk || !kmean || !lse_bias) return ATTN_ERR_ARG;
  if (dtype != ATTN_BF16 && dtype != ATTN_FP16) return ATTN_ERR_ARG;
  if (!std::isfinite(scale)) return ATTN_ERR_ARG;
  int rc = check_shape(B, Hq, Hkv, N, d);
  if (rc) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(q8) || !aligned16(k8) || !aligned16(kmean) || !aligned16(sq) ||
      !aligned16(sk) || !aligned16(lse_bias))
    return ATTN_ERR_ALIGN;
  if (!scratch || scratch_bytes_given < scratch_bytes(B, Hkv, N, d)) return ATTN_ERR_WORKSPACE;
  if (!aligned16(scratch)) return ATTN_ERR_ALIGN;
  return launch_prepass(q, k, B, Hq, Hkv, N, d, dtype, scale, q8, sq, k8, sk, kmean, lse_bias,
                        static_cast<double*>(scratch), static_cast<cudaStream_t>(stream));
}

int attn_quant_smooth_k_noalloc(const void* q, const void* k, int B, int Hq, int Hkv, int N, int d, int dtype,
                                float scale, int8_t* q8, float* sq, int8_t* k8, float* sk, float* kmean,
                                float* lse_bias, void* stream) {
  if (!q || !k || !q8 || !sq || !k8 || !sk || !kmean || !lse_bias) return ATTN_ERR_ARG;
  if (dtype != ATTN_BF16 && dtype != ATTN_FP16) return ATTN_ERR_ARG;
  if (!std::isfinite(scale)) return ATTN_ERR_ARG;
  int rc = check_shape(B, Hq, Hkv, N, d);
  if (rc) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(q8) || !aligned16(k8) || !aligned16(kmean) || !aligned16(sq) ||
      !aligned16(sk) || !aligned16(lse_bias))
    return ATTN_ERR_ALIGN;
  const size_t need = scratch_bytes(B, Hkv, N, d);
  if (need > kStaticScratchBytes) {
    std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error),
                  "these sizes need %zu bytes of K-mean scratch; the built-in scratch holds %zu "
                  "(B*Hkv*ceil(N/128)*d <= %zu); use attn_quant_smooth_k with caller scratch",
                  need, kStaticScratchBytes, kStaticScratchBytes / sizeof(double));
    return ATTN_ERR_WORKSPACE;
  }
  double* part = nullptr;
  if ((rc = static_scratch_address(&part))) return rc;
  // The partials are written in full before they are read, so nothing has to be cleared.
  return launch_prepass(q, k, B, Hq, Hkv, N, d, dtype, scale, q8, sq, k8, sk, kmean, lse_bias, part,
                        static_cast<cudaStream_t>(stream));
}

int attn_fwd_int8_quantized(const int8_t* q8, const float* sq, const int8_t* k8, const float* sk,
                            const float* lse_bias, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int N,
                            int d, int causal, float scale, int dtype, void* stream) {
  int rc = check_common(q8, k8, v, o, lse, B, Hq, Hkv, N, d, causal, scale, dtype);
  if (rc) return rc;
  if (!sq || !sk || (lse && !lse_bias)) return ATTN_ERR_ARG;
  return fwd_quantized(q8, sq, k8, sk, lse_bias, v, o, lse, B, Hq, Hkv, N, d, causal, scale, dtype, false,
                       static_cast<cudaStream_t>(stream));
}

int attn_quant_smooth_k_fp8(const void* q, const void* k, int B, int Hq, int Hkv, int N, int d, int dtype,
                            float scale, uint8_t* q8, float* sq, uint8_t* k8, float* sk, float* kmean,
                            float* lse_bias, void* scratch, size_t scratch_bytes_given, void* stream) {
  if (!q || !k || !q8 || !sq || !k8 || !sk || !kmean || !lse_bias) return ATTN_ERR_ARG;
  if (dtype != ATTN_BF16 && dtype != ATTN_FP16) return ATTN_ERR_ARG;
  if (!std::isfinite(scale)) return ATTN_ERR_ARG;
  int rc = check_shape(B, Hq, Hkv, N, d);
  if (rc) return rc;
  if (!aligned16(q) || !aligned16(k) || !aligned16(q8) || !aligned16(k8) || !aligned16(kmean) || !aligned16(sq) ||
      !aligned16(sk) || !aligned16(lse_bias))
    return ATTN_ERR_ALIGN;
  if (!scratch || scratch_bytes_given < scratch_bytes(B, Hkv, N, d)) return ATTN_ERR_WORKSPACE;
  if (!aligned16(scratch)) return ATTN_ERR_ALIGN;
  return launch_prepass(q, k, B, Hq, Hkv, N, d, dtype, scale, reinterpret_cast<int8_t*>(q8), sq,
                        reinterpret_cast<int8_t*>(k8), sk, kmean, lse_bias, static_cast<double*>(scratch),
                        static_cast<cudaStream_t>(stream), true);
}

int attn_fwd_fp8_quantized(const uint8_t* q8, const float* sq, const uint8_t* k8, const float* sk,
                           const float* lse_bias, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int N,
                           int d, int causal, float scale, int dtype, void* stream) {
  int rc = check_common(q8, k8, v, o, lse, B, Hq, Hkv, N, d, causal, scale, dtype);
  if (rc) return rc;
  if (!sq || !sk || (lse && !lse_bias)) return ATTN_ERR_ARG;
  return fwd_quantized(q8, sq, k8, sk, lse_bias, v, o, lse, B, Hq, Hkv, N, d, causal, scale, dtype, true,
                       static_cast<cudaStream_t>(stream));
}

int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv, int N, int d,
             int causal, float scale, int mode, int dtype, void* workspace, size_t ws_bytes, void* stream) {
  int rc = check_common(q, k, v, o, lse, B, Hq, Hkv, N, d, causal, scale, dtype);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (mode == ATTN_MODE_BF16_EXACT) {
    FwdParams p = make_params(B, Hq, Hkv, N, causal, scale, o, lse);
    return launch_fwd<QK_F16>(q, k, v, d, dtype, p, st);
  }
  if (mode != ATTN_MODE_INT8_QK && mode != ATTN_MODE_FP8_QK) return ATTN_ERR_ARG;
  const bool f8 = mode == ATTN_MODE_FP8_QK;
  const WsLayout w = ws_layout(B, Hq, Hkv, N, d);
  if (!workspace || ws_bytes < w.total) return ATTN_ERR_WORKSPACE;
  if (!aligned16(workspace)) return ATTN_ERR_ALIGN;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  auto* q8 = reinterpret_cast<int8_t*>(ws + w.q8);
  auto* k8 = reinterpret_cast<int8_t*>(ws + w.k8);
  auto* sq = reinterpret_cast<float*>(ws + w.sq);
  auto* sk = reinterpret_cast<float*>(ws + w.sk);
  auto* kmean = reinterpret_cast<float*>(ws + w.kmean);
  auto* bias = reinterpret_cast<float*>(ws + w.bias);
  auto* part = reinterpret_cast<double*>(ws + w.scratch);
  rc = launch_prepass(q, k, B, Hq, Hkv, N, d, dtype, scale, q8, sq, k8, sk, kmean, bias, part, st, f8);
  if (rc) return rc;
  return fwd_quantized(q8, sq, k8, sk, bias, v, o, lse, B, Hq, Hkv, N, d, causal, scale, dtype, f8, st);
}

int attn_probe_qk_int32(const int8_t* q8, const int8_t* k8, int B, int Hq, int Hkv, int N, int d,
                        const int32_t* tiles, int ntiles, int32_t* out, void* stream) {
  if (!q8 || !k8 || !tiles || !out || ntiles < 1) return ATTN_ERR_ARG;
  int rc = check_shape(B, Hq, Hkv, N, d);
  if (rc) return rc;
  if (!aligned16(q8) || !aligned16(k8) || !aligned16(out) || !aligned16(tiles)) return ATTN_ERR_ALIGN;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  CUtensorMap tq, tk;
  const int row = d;  // int8 row bytes
  const int box_x = row >= 128 ? 128 : 64;
  if ((rc = make_map(&tq, q8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, d, N, B * Hq, box_x, swizzle_for(row)))) return rc;
  if ((rc = make_map(&tk, k8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, d, N, B * Hkv, box_x, swizzle_for(row)))) return rc;
  const int smem = 2 * 128 * d + 64 + 1024;
  if (d == 128) {
    probe_qk_kernel<128><<<ntiles, 160, smem, st>>>(tq, tk, B, Hq, Hkv, N, tiles, out);
  } else {
    probe_qk_kernel<64><<<ntiles, 160, smem, st>>>(tq, tk, B, Hq, Hkv, N, tiles, out);
  }
  TATTN_CUDA(cudaGetLastError());
  return ATTN_OK;
}

// The pieces attn_fwd_host cuts B*Hq query heads into, as cut points cut[0] = 0 < cut[1] < ... <
// cut[n] = B*Hq (n <= kMaxPieces, returned).  A piece is either whole (batch, kv head) units
// (G = Hq/Hkv heads each) or a run of query heads inside one unit.  When N % 4 == 0 (every
// head's lse slice 16-byte aligned) the first and last pieces are one query head each (one unit
// when G = 1) and the units between form up to six pieces; otherwise up to 8 runs of whole
// units, 4-unit aligned when a unit's lse slice is not 16-byte aligned.
constexpr int kMaxPieces = 16;
static int host_pieces(int B, int Hq, int Hkv, int N, int* cut) {
  const int G = Hq / Hkv;
  const int units = B * Hkv, heads = B * Hq;
  int c[kMaxPieces + 8];
  int nc = 0;
  if (N % 4 == 0) {
    c[nc++] = 0;
    c[nc++] = 1;
    c[nc++] = G;
    const int mid = units - 2 > 0 ? units - 2 : 0;  // units strictly between the first and last
    const int nm = mid < 6 ? mid : 6;
    for (int i = 1; i < nm; ++i) c[nc++] = (1 + (int)((long long)mid * i / nm)) * G;
    c[nc++] = heads - G;
    c[nc++] = heads - 1;
    c[nc++] = heads;
  } else {
    const int align_units = ((size_t)G * N * 4 % 16 == 0) ? 1 : 4;
    const int n8 = units < 8 ? units : 8;
    for (int i = 0; i <= n8; ++i) c[nc++] = (int)((long long)units * i / n8) / align_units * align_units * G;
    c[nc++] = heads;
  }
  std::sort(c, c + nc);
  int n = 0;
  for (int i = 0; i < nc; ++i) {
    if (i > 0 && c[i] == c[i - 1]) continue;
    cut[n++] = c[i];
  }
  return n - 1;
}

int attn_fwd_host(const void* q, const void* k, const void* v, void* o, float* lse, void* dq, void* dk, void* dv,
                  void* do_, float* dlse, int B, int Hq, int Hkv, int N, int d, int causal, float scale, int mode,
                  int dtype, void* workspace, size_t ws_bytes, void* stream) {
  if (!q || !k || !v || !o) return ATTN_ERR_ARG;
  int rc = check_common(dq, dk, dv, do_, dlse, B, Hq, Hkv, N, d, causal, scale, dtype);
  if (rc) return rc;
  if (mode != ATTN_MODE_BF16_EXACT && mode != ATTN_MODE_INT8_QK && mode != ATTN_MODE_FP8_QK) return ATTN_ERR_ARG;
  if (mode != ATTN_MODE_BF16_EXACT && (!workspace || ws_bytes < attn_workspace_bytes(B, Hq, Hkv, N, d, mode)))
    return ATTN_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const bool want_lse = lse && dlse;
  // Units are (batch, kv head) pairs with their G query heads: independent problems whose Q, K, V,
  // O and lse slices are contiguous, in unit order, in every [B, H, N, d] tensor.  A run of whole
  // units is one problem with B' = 1, Hq' = n*G, Hkv' = n, and a run of query heads inside one
  // unit is one with B' = 1, Hq' = n, Hkv' = 1 (the unit's K and V); either gives every output row
  // the same arithmetic as the whole call.  The work is cut into pieces of query heads
  // (host_pieces); piece c's inputs are copied in on a helper stream while piece c-1 computes on
  // the caller's stream, and its outputs are copied out on a second helper stream.  Only the first
  // piece's input copy and the last piece's output copy are not hidden behind compute, which is
  // why those two pieces are kept small.
  const int G = Hq / Hkv;
  const size_t q_head = (size_t)N * d * 2, kv_unit = (size_t)N * d * 2, l_head = (size_t)N * 4;
  int cut[kMaxPieces + 1];
  const int npiece = host_pieces(B, Hq, Hkv, N, cut);
  cudaStream_t s_in = nullptr, s_out = nullptr;
  cudaEvent_t ev_in[kMaxPieces] = {}, ev_done[kMaxPieces] = {};
  auto cleanup = [&]() {
    for (int c = 0; c < kMaxPieces; ++c) {
      if (ev_in[c]) cudaEventDestroy(ev_in[c]);
      if (ev_done[c]) cudaEventDestroy(ev_done[c]);
    }
    if (s_in) cudaStreamDestroy(s_in);
    if (s_out) cudaStreamDestroy(s_out);
  };
#define TATTN_CUDA_C(call)                          \
  do {                                              \
    cudaError_t e_ = (call);                        \
    if (e_ != cudaSuccess) {                        \
      cleanup();                                    \
      return cuda_fail(e_, #call);                  \
    }                                               \
  } while (0)
  TATTN_CUDA_C(cudaStreamCreateWithFlags(&s_in, cudaStreamNonBlocking));
  TATTN_CUDA_C(cudaStreamCreateWithFlags(&s_out, cudaStreamNonBlocking));
  for (int c = 0; c < npiece; ++c) {
    TATTN_CUDA_C(cudaEventCreateWithFlags(&ev_in[c], cudaEventDisableTiming));
    TATTN_CUDA_C(cudaEventCreateWithFlags(&ev_done[c], cudaEventDisableTiming));
  }
  // inputs may still be in use by earlier work on the caller's stream: start after it
  TATTN_CUDA_C(cudaEventRecord(ev_done[0], st));
  TATTN_CUDA_C(cudaStreamWaitEvent(s_in, ev_done[0], 0));
  auto copy_in = [&](size_t off, size_t bytes, void* dst, const void* src) {
    return cudaMemcpyAsync(static_cast<uint8_t*>(dst) + off, static_cast<const uint8_t*>(src) + off, bytes,
                           cudaMemcpyHostToDevice, s_in);
  };
  for (int c = 0; c < npiece; ++c) {
    const int h0 = cut[c], h1 = cut[c + 1];
    TATTN_CUDA_C(copy_in(h0 * q_head, (size_t)(h1 - h0) * q_head, dq, q));
    // K and V of every unit this piece starts (a piece inside a unit that another piece started
    // reuses them)
    const int u0 = (h0 + G - 1) / G, u1 = (h1 + G - 1) / G;
    if (u1 > u0) {
      TATTN_CUDA_C(copy_in(u0 * kv_unit, (size_t)(u1 - u0) * kv_unit, dk, k));
      TATTN_CUDA_C(copy_in(u0 * kv_unit, (size_t)(u1 - u0) * kv_unit, dv, v));
    }
    TATTN_CUDA_C(cudaEventRecord(ev_in[c], s_in));
  }
  for (int c = 0; c < npiece; ++c) {
    const int h0 = cut[c], h1 = cut[c + 1];
    const bool whole = h0 % G == 0 && (h1 - h0) % G == 0;
    const int hq = h1 - h0, hkv = whole ? hq / G : 1, ukv = h0 / G;
    TATTN_CUDA_C(cudaStreamWaitEvent(st, ev_in[c], 0));
    rc = attn_fwd(static_cast<uint8_t*>(dq) + h0 * q_head, static_cast<uint8_t*>(dk) + ukv * kv_unit,
                  static_cast<uint8_t*>(dv) + ukv * kv_unit, static_cast<uint8_t*>(do_) + h0 * q_head,
                  want_lse ? reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(dlse) + h0 * l_head) : nullptr, 1,
                  hq, hkv, N, d, causal, scale, mode, dtype, workspace, ws_bytes, stream);
    if (rc) {
      cudaStreamSynchronize(s_in);
      cudaStreamSynchronize(st);
      cleanup();
      return rc;
    }
    TATTN_CUDA_C(cudaEventRecord(ev_done[c], st));
    TATTN_CUDA_C(cudaStreamWaitEvent(s_out, ev_done[c], 0));
    TATTN_CUDA_C(cudaMemcpyAsync(static_cast<uint8_t*>(o) + h0 * q_head, static_cast<uint8_t*>(do_) + h0 * q_head,
                                 (size_t)hq * q_head, cudaMemcpyDeviceToHost, s_out));
    if (want_lse)
      TATTN_CUDA_C(cudaMemcpyAsync(reinterpret_cast<uint8_t*>(lse) + h0 * l_head,
                                   reinterpret_cast<uint8_t*>(dlse) + h0 * l_head, (size_t)hq * l_head,
                                   cudaMemcpyDeviceToHost, s_out));
  }
  TATTN_CUDA_C(cudaStreamSynchronize(s_out));
  TATTN_CUDA_C(cudaStreamSynchronize(st));
#undef TATTN_CUDA_C
  cleanup();
  return ATTN_OK;
}

int attn_fwd_prefix_masked(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                           int Nq, int Nk, int d, const int32_t* row_kv_limit, float scale, int dtype, void* stream) {
  int rc = check_common(q, k, v, o, lse, B, Hq, Hkv, Nq, d, 0, scale, dtype);
  if (rc) return rc;
  if (Nk < 1 || !row_kv_limit) return ATTN_ERR_ARG;
  if ((rc = check_shape(B, Hq, Hkv, Nk, d))) return rc;
  if (reinterpret_cast<uintptr_t>(row_kv_limit) & 3u) return ATTN_ERR_ALIGN;
  if (TATTN_SPLIT) return ATTN_ERR_UNSUPPORTED;  // the four-threads-per-row variant has no row limits
  FwdParams p = make_params(B, Hq, Hkv, Nq, 0, scale, o, lse, Nk, row_kv_limit);
  return launch_fwd<QK_F16>(q, k, v, d, dtype, p, static_cast<cudaStream_t>(stream));
}

size_t attn_decode_workspace_bytes(int B, int Hq, int Hkv, int Nq, int Nk, int d, int num_ctas) {
  if (check_decode_shape(B, Hq, Hkv, Nq, Nk, d, num_ctas)) return 0;
  return decode_ws(B, Hkv, (Hq / Hkv) * Nq, decode_ctas(B, Hkv, Nk, num_ctas)).total;
}

int attn_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* kv_lens, void* o, float* lse,
                int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal, float scale, int dtype, int num_ctas,
                void* workspace, size_t ws_bytes, void* stream) {
  if (!q || !k_cache || !v_cache || !o) return ATTN_ERR_ARG;
  if (causal != 0 && causal != 1) return ATTN_ERR_ARG;
  if (!std::isfinite(scale) || !(scale > 0.f)) return ATTN_ERR_ARG;
  if (dtype != ATTN_BF16 && dtype != ATTN_FP16) return ATTN_ERR_ARG;
  int rc = check_decode_shape(B, Hq, Hkv, Nq, Nk, d, num_ctas);
  if (rc) return rc;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o) || (lse && !aligned16(lse)) ||
      (reinterpret_cast<uintptr_t>(kv_lens) & 3u))
    return ATTN_ERR_ALIGN;
  const int R = (Hq / Hkv) * Nq;
  const int ctas = decode_ctas(B, Hkv, Nk, num_ctas);
  const DecWs w = decode_ws(B, Hkv, R, ctas);
  if (!workspace || ws_bytes < w.total) return ATTN_ERR_WORKSPACE;
  if (!aligned16(workspace)) return ATTN_ERR_ALIGN;
  DecParams p{};
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Nq = Nq;
  p.Nk = Nk;
  p.R = R;
  p.causal = causal;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.kv_lens = kv_lens;
  p.o = o;
  p.lse = lse;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  p.part_o = reinterpret_cast<float*>(ws + w.part_o);
  p.part_lse = reinterpret_cast<float*>(ws + w.part_lse);
  p.unit_arrived = reinterpret_cast<unsigned int*>(ws + w.unit_arrived);
  return launch_decode(q, k_cache, v_cache, dtype, ctas, p, static_cast<cudaStream_t>(stream));
}

int attn_merge_lse(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part, void* o_out,
                   long long rows, int d, int dtype, int first, void* stream) {
  if (!o_acc || !lse_acc || rows < 0 || (first != 0 && first != 1)) return ATTN_ERR_ARG;
  if (first && (!o_part || !lse_part)) return ATTN_ERR_ARG;
  if ((o_part == nullptr) != (lse_part == nullptr)) return ATTN_ERR_ARG;
  if (dtype != ATTN_BF16 && dtype != ATTN_FP16) return ATTN_ERR_ARG;
  if (d != 64 && d != 128) return ATTN_ERR_UNSUPPORTED;
  if (!aligned16(o_acc) || !aligned16(lse_acc) || (o_part && !aligned16(o_part)) ||
      (lse_part && !aligned16(lse_part)) || (o_out && !aligned16(o_out)))
    return ATTN_ERR_ALIGN;
  if (rows == 0) return ATTN_OK;
  const long long want = (rows + 7) / 8;  // 8 rows (one per warp) per CTA of 256 threads
  const unsigned grid = (unsigned)std::min<long long>(want, (long long)device_sm_count() * 16);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const auto* part = static_cast<const uint16_t*>(o_part);
  auto* out = static_cast<uint16_t*>(o_out);
  const bool fp16 = dtype == ATTN_FP16;
  if (d == 128) {
    if (fp16) lse_merge_kernel<128, true><<<grid, 256, 0, st>>>(o_acc, lse_acc, part, lse_part, out, rows, first);
    else lse_merge_kernel<128, false><<<grid, 256, 0, st>>>(o_acc, lse_acc, part, lse_part, out, rows, first);
  } else {
    if (fp16) lse_merge_kernel<64, true><<<grid, 256, 0, st>>>(o_acc, lse_acc, part, lse_part, out, rows, first);
    else lse_merge_kernel<64, false><<<grid, 256, 0, st>>>(o_acc, lse_acc, part, lse_part, out, rows, first);
  }
  TATTN_CUDA(cudaGetLastError());
  return ATTN_OK;
}

int attn_check_status(void) {
  TATTN_CUDA(cudaDeviceSynchronize());
  int st = 0, zero = 0;
  TATTN_CUDA(cudaMemcpyFromSymbol(&st, tattn::g_status, sizeof(int)));
  TATTN_CUDA(cudaMemcpyToSymbol(tattn::g_status, &zero, sizeof(int)));
  return (st & tattn::STATUS_TIMEOUT) ? ATTN_ERR_TIMEOUT : ATTN_OK;
}

// Test hook for failure detection: one thread waits on an mbarrier that nothing ever completes,
// with a limit of `limit_us` microseconds, so the bounded-wait path runs without faulting the GPU.
int attn_test_host_pieces(int B, int Hq, int Hkv, int N, int d, int* cuts, int max_cuts) {
  if (!cuts || max_cuts < kMaxPieces + 1) return ATTN_ERR_ARG;
  int rc = check_shape(B, Hq, Hkv, N, d);
  if (rc) return rc;
  return host_pieces(B, Hq, Hkv, N, cuts);
}

int attn_test_wait_timeout(int limit_us, void* stream) {
  if (limit_us < 1 || limit_us > 1000000) return ATTN_ERR_ARG;
  wait_forever_probe_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>((unsigned long long)limit_us * 1000ull);
  TATTN_CUDA(cudaGetLastError());
  return ATTN_OK;
}

// Test hook: the fused kernel's exp2 routines applied to an array (1 = FMA-pipe polynomial,
// 0 = MUFU ex2.approx), so tests can compare them with CUDA's exp2f.
int attn_test_exp2(const float* x, float* y, int n, int use_poly, void* stream) {
  if (!x || !y || n < 1) return ATTN_ERR_ARG;
  exp2_eval_kernel<<<(n + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n, use_poly);
  TATTN_CUDA(cudaGetLastError());
  return ATTN_OK;
}

const char* attn_error_string(int code) {
  switch (code) {
    case ATTN_OK: return "ok";
    case ATTN_ERR_ARG: return "invalid argument";
    case ATTN_ERR_UNSUPPORTED: return "unsupported size (d must be 64 or 128; decode: d = 128, (Hq/Hkv)*Nq <= 64)";
    case ATTN_ERR_ALIGN: return "device pointer not 16-byte aligned";
    case ATTN_ERR_WORKSPACE: return "workspace missing or too small";
    case ATTN_ERR_LAUNCH: return "CUDA launch or call failed";
    case ATTN_ERR_TIMEOUT: return "a device-side wait timed out";
    default: return "unknown status";
  }
}

const char* attn_last_cuda_error(void) { return g_last_cuda_error; }

}  // extern "C"
