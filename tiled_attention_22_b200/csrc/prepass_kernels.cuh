// prepass_kernels.cuh - the INT8 pre-pass of the SageAttention-style mode, for sm_100a.
//
// SageAttention article ("又快又准，即插即用！清华8比特量化Attention…", section 技术方案):
//   (1) K is smoothed by removing its mean over tokens from every key, which leaves
//       softmax(Q K^T) unchanged;
//   (2) Q and K are quantised to INT8 with one scale per block of the attention tiling.
// Readings fixed by this library (the article's algorithm figure did not survive): the mean is per
// (batch, kv head, channel) over all N tokens; blocks are 128 tokens x all d channels; scale =
// amax/127, code = clamp(rint(x * (127/amax)), -127, 127) with ties to even; a zero block gets scale 0.
//
// These kernels are HBM-bound: plain 16-byte vector loads and stores, no tensor cores.
//   kmean_partial_kernel  K -> float64 partial sums per 128-token block (sequential in token order)
//   kmean_final_kernel    partials -> mean (sequential in block order), (float)(total / N)
//   quant_kernel          K blocks: smooth + quantise -> k8, sk;  Q blocks: quantise -> q8, sq and
//                         the lse bias scale * q_i . mean (row dot product, warp-shuffle reduced)
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

namespace tattn {

template <bool FP16>
__device__ __forceinline__ void unpack8(const uint4& v, float (&x)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if constexpr (FP16) {
      __half2 h = *reinterpret_cast<const __half2*>(&w[i]);
      float2 f = __half22float2(h);
      x[2 * i] = f.x;
      x[2 * i + 1] = f.y;
    } else {
      __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(&w[i]);
      float2 f = __bfloat1622float2(h);
      x[2 * i] = f.x;
      x[2 * i + 1] = f.y;
    }
  }
}

// One thread = one (batch*kv head, 128-token block, 8-channel chunk).  Adds the block's tokens in
// ascending order into float64 accumulators (one per channel), starting from 0.0.
template <bool FP16>
__global__ void __launch_bounds__(128) kmean_partial_kernel(const uint16_t* __restrict__ k, int BG, int N, int d,
                                                             double* __restrict__ part) {
  const int chunks = d / 8;
  const int T = (N + 127) / 128;
  const long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (long long)BG * T * chunks) return;
  const int chunk = (int)(idx % chunks);
  const long long rest = idx / chunks;
  const int t = (int)(rest % T);
  const int bg = (int)(rest / T);
  const int cnt = min(128, N - t * 128);
  const uint4* src = reinterpret_cast<const uint4*>(k + ((size_t)bg * N + (size_t)t * 128) * d + chunk * 8);
  const int stride = d / 8;  // uint4 per row
  double acc[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) acc[c] = 0.0;
  int i = 0;
  for (; i + 8 <= cnt; i += 8) {
    uint4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = __ldg(src + (size_t)(i + u) * stride);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      float x[8];
      unpack8<FP16>(v[u], x);
#pragma unroll
      for (int c = 0; c < 8; ++c) acc[c] = __dadd_rn(acc[c], (double)x[c]);
    }
  }
  for (; i < cnt; ++i) {
    float x[8];
    unpack8<FP16>(__ldg(src + (size_t)i * stride), x);
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[c] = __dadd_rn(acc[c], (double)x[c]);
  }
  double* dst = part + ((size_t)bg * T + t) * d + chunk * 8;
#pragma unroll
  for (int c = 0; c < 8; ++c) dst[c] = acc[c];
}

// One thread = one (batch*kv head, channel): total over blocks in ascending order, then the mean.
__global__ void __launch_bounds__(128) kmean_final_kernel(const double* __restrict__ part, int BG, int N, int d,
                                                           float* __restrict__ kmean) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= BG * d) return;
  const int bg = idx / d, c = idx % d;
  const int T = (N + 127) / 128;
  const double* src = part + (size_t)bg * T * d + c;
  double total = 0.0;
  for (int t = 0; t < T; ++t) total = __dadd_rn(total, src[(size_t)t * d]);
  kmean[idx] = __double2float_rn(__ddiv_rn(total, (double)N));
}

// 256 threads per CTA, one CTA per 128-token block.  Blocks [0, nK) are K blocks (b, g, t),
// blocks [nK, nK + nQ) are Q blocks (b, h, t).  Thread layout: d/16 threads per row, each holding
// 16 consecutive channels; rows are covered in passes of 256 / (d/16) rows.
template <int D, bool FP16>
__global__ void __launch_bounds__(256) quant_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                                                     int B, int Hq, int Hkv, int N, float scale,
                                                     const float* __restrict__ kmean, int8_t* __restrict__ q8,
                                                     float* __restrict__ sq, int8_t* __restrict__ k8,
                                                     float* __restrict__ sk, float* __restrict__ bias) {
  constexpr int TPR = D / 16;           // threads per row
  constexpr int RPP = 256 / TPR;        // rows per pass
  constexpr int PASSES = 128 / RPP;
  __shared__ float warp_max[8];

  const int T = (N + 127) / 128;
  const int nK = B * Hkv * T;
  const bool is_k = (int)blockIdx.x < nK;
  const int blk = is_k ? blockIdx.x : blockIdx.x - nK;
  const int t = blk % T;
  const int bh = blk / T;  // b*Hkv + g for K, b*Hq + h for Q
  const int g_mean = is_k ? bh : (bh / Hq) * Hkv + (bh % Hq) / (Hq / Hkv);
  const uint16_t* src = (is_k ? k : q) + ((size_t)bh * N + (size_t)t * 128) * D;
  int8_t* dst = (is_k ? k8 : q8) + ((size_t)bh * N + (size_t)t * 128) * D;
  const int cnt = min(128, N - t * 128);
  const int tid = threadIdx.x;
  const int chunk = tid % TPR, r_in = tid / TPR;

  float mean[16];
  {
    const float4* m4 = reinterpret_cast<const float4*>(kmean + (size_t)g_mean * D + chunk * 16);
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const float4 m = __ldg(m4 + v);
      mean[4 * v] = m.x;
      mean[4 * v + 1] = m.y;
      mean[4 * v + 2] = m.z;
      mean[4 * v + 3] = m.w;
    }
  }

  float x[PASSES][16];
  float amax = 0.f;
#pragma unroll
  for (int ps = 0; ps < PASSES; ++ps) {
    const int row = ps * RPP + r_in;
    const bool valid = row < cnt;  // uniform over the TPR lanes of one row
    if (valid) {
      const uint4* s4 = reinterpret_cast<const uint4*>(src + (size_t)row * D + chunk * 16);
      float lo[8], hi[8];
      unpack8<FP16>(__ldg(s4), lo);
      unpack8<FP16>(__ldg(s4 + 1), hi);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        x[ps][c] = lo[c];
        x[ps][8 + c] = hi[c];
      }
      if (is_k) {
#pragma unroll
        for (int c = 0; c < 16; ++c) x[ps][c] = __fsub_rn(x[ps][c], mean[c]);
      }
    } else {
#pragma unroll
      for (int c = 0; c < 16; ++c) x[ps][c] = 0.f;
    }
    if (!is_k) {  // CTA-uniform branch
      // lse bias: scale * q_row . mean; 16 channels per lane, then a shuffle sum over the row's lanes
      float dot = 0.f;
#pragma unroll
      for (int c = 0; c < 16; ++c) dot = fmaf(x[ps][c], mean[c], dot);
#pragma unroll
      for (int off = TPR / 2; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
      if (valid && chunk == 0) bias[(size_t)bh * N + (size_t)t * 128 + row] = scale * dot;
    }
#pragma unroll
    for (int c = 0; c < 16; ++c) amax = fmaxf(amax, fabsf(x[ps][c]));
  }
  // block absmax: warp shuffle, then across the 8 warps
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  if ((tid & 31) == 0) warp_max[tid >> 5] = amax;
  __syncthreads();
  amax = warp_max[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) amax = fmaxf(amax, warp_max[w]);

  const bool zero = (amax == 0.f);
  const float scl = zero ? 0.f : __fdiv_rn(amax, 127.0f);
  const float inv = zero ? 0.f : __fdiv_rn(127.0f, amax);
  if (tid == 0) (is_k ? sk : sq)[(size_t)bh * T + t] = scl;

#pragma unroll
  for (int ps = 0; ps < PASSES; ++ps) {
    const int row = ps * RPP + r_in;
    if (row < cnt) {
      uint32_t w[4];
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        uint32_t packed = 0;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          int code = 0;
          if (!zero) {
            code = __float2int_rn(__fmul_rn(x[ps][4 * v + c], inv));
            code = max(-127, min(127, code));
          }
          packed |= (uint32_t)(code & 0xff) << (8 * c);
        }
        w[v] = packed;
      }
      *reinterpret_cast<uint4*>(dst + (size_t)row * D + chunk * 16) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

}  // namespace tattn
