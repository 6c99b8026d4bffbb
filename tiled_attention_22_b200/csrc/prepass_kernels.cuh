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
//   kmean_partial_kernel  K -> float64 partial sums per 128-token block (sequential in token order,
//                         the block staged in shared memory)
//   kmean_final_kernel    partials -> mean (sequential in block order), (float)(total / N); the
//                         partials stream through shared memory (cp.async pipeline)
//   quant_kernel          K blocks: smooth + quantise -> k8, sk;  Q blocks: quantise -> q8, sq and
//                         the lse bias scale * q_i . mean (row dot product, warp-shuffle reduced)
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

namespace tattn {

// max(a, |b|, |c|) in one instruction
__device__ __forceinline__ float max3_abs(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(fabsf(b)), "f"(fabsf(c)));
  return d;
}

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

// One CTA (D threads) per (batch*kv head, 128-token block): the block is staged in shared memory
// with 16-byte loads (whole rows, so each DRAM page is read in one sweep), then thread c adds
// channel c's tokens in ascending order into a float64 partial starting at 0.0.
template <int D, bool FP16>
__global__ void __launch_bounds__(D) kmean_partial_kernel(const uint16_t* __restrict__ k, int N,
                                                           double* __restrict__ part) {
  __shared__ __align__(16) uint16_t tile[128 * D];
  const int T = (N + 127) / 128;
  const int t = blockIdx.x % T;
  const int bg = blockIdx.x / T;
  const int cnt = min(128, N - t * 128);
  const uint4* src = reinterpret_cast<const uint4*>(k + ((size_t)bg * N + (size_t)t * 128) * D);
  uint4* dst = reinterpret_cast<uint4*>(tile);
  const int n16 = cnt * D / 8;  // 16-byte chunks in the block
#pragma unroll 4
  for (int i = threadIdx.x; i < n16; i += D) dst[i] = __ldg(src + i);
  __syncthreads();
  const int c = threadIdx.x;
  double acc = 0.0;
  for (int i = 0; i < cnt; ++i) {
    const uint16_t b = tile[i * D + c];
    float x;
    if constexpr (FP16)
      x = __half2float(__ushort_as_half(b));
    else
      x = __uint_as_float((uint32_t)b << 16);
    acc = __dadd_rn(acc, (double)x);
  }
  part[((size_t)bg * T + t) * D + c] = acc;
}

// One CTA per (batch * kv head): thread c < D adds channel c's block partials in ascending block
// order into a float64 total, then writes (float)(total / N).  The partials of one (batch, kv head)
// ([T][D] float64, contiguous) stream through shared memory in chunks of kFinalChunk blocks with
// cp.async, kFinalStages - 1 chunks in flight, so the sequential adds never wait on a global load.
constexpr int kFinalThreads = 512;
constexpr int kFinalChunk = 16;
constexpr int kFinalStages = 8;
template <int D>
constexpr int kmean_final_smem() { return kFinalStages * kFinalChunk * D * (int)sizeof(double); }

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(smem_dst)),
               "l"(gmem_src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <int D>
__global__ void __launch_bounds__(kFinalThreads) kmean_final_kernel(const double* __restrict__ part, int N,
                                                                     float* __restrict__ kmean) {
  extern __shared__ __align__(16) double fbuf[];  // [kFinalStages][kFinalChunk * D]
  constexpr int CHUNK = kFinalChunk * D;        // doubles per chunk
  const int bg = blockIdx.x;
  const int T = (N + 127) / 128;
  const double* src = part + (size_t)bg * T * D;
  const int total_elems = T * D;
  const int nchunk = (T + kFinalChunk - 1) / kFinalChunk;
  // chunk k -> stage k % kFinalStages; each thread copies 16-byte pieces (two partials)
  auto issue = [&](int k) {
    if (k < nchunk) {
      double* dst = fbuf + (k % kFinalStages) * CHUNK;
      const int base = k * CHUNK;
      for (int e = 2 * threadIdx.x; e < CHUNK; e += 2 * kFinalThreads)
        if (base + e < total_elems) cp_async16(dst + e, src + base + e);
    }
    cp_async_commit();  // one group per chunk (empty past the end), so group counts stay aligned
  };
#pragma unroll 1
  for (int k = 0; k < kFinalStages - 1; ++k) issue(k);
  double total = 0.0;
#pragma unroll 1
  for (int k = 0; k < nchunk; ++k) {
    cp_async_wait<kFinalStages - 2>();  // chunk k has landed (this thread's copies)
    __syncthreads();                    // ... and every other thread's
    if (threadIdx.x < D) {
      const double* b = fbuf + (k % kFinalStages) * CHUNK + threadIdx.x;
      const int nt = min(kFinalChunk, T - k * kFinalChunk);
      for (int t = 0; t < nt; ++t) total = __dadd_rn(total, b[t * D]);
    }
    __syncthreads();                    // stage k % kFinalStages is free again
    issue(k + kFinalStages - 1);
  }
  cp_async_wait<0>();
  if (threadIdx.x < D) kmean[(size_t)bg * D + threadIdx.x] = __double2float_rn(__ddiv_rn(total, (double)N));
}

// One CTA per 128-token block (4*D threads: 512 for d=128, 256 for d=64).  Blocks [0, nK) are K
// blocks (b, g, t), blocks [nK, nK + nQ) are Q blocks (b, h, t).  Thread layout: d/8 threads per
// row, each holding 8 consecutive channels (one 16-byte load per row); rows are covered in
// 4 passes of 32 rows.  The block stays in registers as raw 16-bit pairs; it is unpacked once for
// the absmax (and Q's bias dot product) and again for quantisation, which keeps the register
// count at 64 (1024 resident threads per SM, 64 KB of loads in flight).
template <int D>
constexpr int quant_threads() { return 4 * D; }

// Two float32 values to two E4M3 codes (round to nearest even, saturating at +-448): lo in the
// low byte, hi in the high byte.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// F8: FP8 (E4M3) codes with scale amax/448 instead of INT8 codes with scale amax/127.
template <int D, bool FP16, bool F8>
__global__ void __launch_bounds__(4 * D, 256 / D) quant_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                                                        int B, int Hq, int Hkv, int N, float scale,
                                                        const float* __restrict__ kmean, int8_t* __restrict__ q8,
                                                        float* __restrict__ sq, int8_t* __restrict__ k8,
                                                        float* __restrict__ sk, float* __restrict__ bias) {
  constexpr int NT = 4 * D;
  constexpr int TPR = D / 8;            // threads per row
  constexpr int RPP = NT / TPR;         // rows per pass (32)
  constexpr int PASSES = 128 / RPP;     // 4
  constexpr int NW = NT / 32;
  __shared__ float warp_max[NW];

  const int T = (N + 127) / 128;
  const int nK = B * Hkv * T;
  const bool is_k = (int)blockIdx.x < nK;
  // K blocks run last-to-first: the mean pass just streamed K first-to-last, so the end of K is
  // what is still in L2 (K is often about the size of L2) and is read again first.
#ifndef TATTN_QUANT_K_REVERSE
#define TATTN_QUANT_K_REVERSE 1
#endif
  const int blk = is_k ? (TATTN_QUANT_K_REVERSE ? nK - 1 - (int)blockIdx.x : (int)blockIdx.x) : (int)blockIdx.x - nK;
  const int t = blk % T;
  const int bh = blk / T;  // b*Hkv + g for K, b*Hq + h for Q
  const int g_mean = is_k ? bh : (bh / Hq) * Hkv + (bh % Hq) / (Hq / Hkv);
  const uint16_t* src = (is_k ? k : q) + ((size_t)bh * N + (size_t)t * 128) * D;
  int8_t* dst = (is_k ? k8 : q8) + ((size_t)bh * N + (size_t)t * 128) * D;
  const int cnt = min(128, N - t * 128);
  const int tid = threadIdx.x;
  const int chunk = tid % TPR, r_in = tid / TPR;

  float mean[8];
  {
    const float4* m4 = reinterpret_cast<const float4*>(kmean + (size_t)g_mean * D + chunk * 8);
    const float4 a = __ldg(m4), b = __ldg(m4 + 1);
    mean[0] = a.x; mean[1] = a.y; mean[2] = a.z; mean[3] = a.w;
    mean[4] = b.x; mean[5] = b.y; mean[6] = b.z; mean[7] = b.w;
  }

  float x[PASSES][8];
  {
    uint4 raw[PASSES];
#pragma unroll
    for (int ps = 0; ps < PASSES; ++ps) {
      const int row = ps * RPP + r_in;
      raw[ps] = row < cnt ? __ldg(reinterpret_cast<const uint4*>(src + (size_t)row * D + chunk * 8))
                          : make_uint4(0, 0, 0, 0);  // +0.0 in both 16-bit formats
    }
#pragma unroll
    for (int ps = 0; ps < PASSES; ++ps) unpack8<FP16>(raw[ps], x[ps]);
  }
  float amax = 0.f;
#pragma unroll
  for (int ps = 0; ps < PASSES; ++ps) {
    const int row = ps * RPP + r_in;
    const bool valid = row < cnt;  // uniform over the TPR lanes of one row
    if (is_k) {
#pragma unroll
      for (int c = 0; c < 8; ++c) x[ps][c] = valid ? __fsub_rn(x[ps][c], mean[c]) : 0.f;
    } else {  // CTA-uniform branch
      // lse bias: scale * q_row . mean; 8 channels per lane, then a shuffle sum over the row's lanes
      float dot = 0.f;
#pragma unroll
      for (int c = 0; c < 8; ++c) dot = fmaf(x[ps][c], mean[c], dot);
#pragma unroll
      for (int off = TPR / 2; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
      if (valid && chunk == 0) bias[(size_t)bh * N + (size_t)t * 128 + row] = scale * dot;
    }
#pragma unroll
    for (int c = 0; c < 8; c += 2) amax = max3_abs(amax, x[ps][c], x[ps][c + 1]);
  }
  // block absmax: warp shuffle, then across the warps
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  if ((tid & 31) == 0) warp_max[tid >> 5] = amax;
  __syncthreads();
  amax = warp_max[0];
#pragma unroll
  for (int w = 1; w < NW; ++w) amax = fmaxf(amax, warp_max[w]);

  const bool zero = (amax == 0.f);
  constexpr float QMAX = F8 ? 448.0f : 127.0f;  // largest code magnitude
  const float scl = zero ? 0.f : __fdiv_rn(amax, QMAX);
  const float inv = zero ? 0.f : __fdiv_rn(QMAX, amax);
  if (tid == 0) (is_k ? sk : sq)[(size_t)bh * T + t] = scl;

  if constexpr (F8) {
    // code = E4M3(fl(x * inv)); |fl(x * inv)| <= 448 (1 + 2^-23), which rounds to 448 at most
#pragma unroll
    for (int ps = 0; ps < PASSES; ++ps) {
      const int row = ps * RPP + r_in;
      if (row < cnt) {
        uint32_t h[4];
#pragma unroll
        for (int c = 0; c < 4; ++c)
          h[c] = e4m3x2(__fmul_rn(x[ps][2 * c], inv), __fmul_rn(x[ps][2 * c + 1], inv));
        *reinterpret_cast<uint2*>(dst + (size_t)row * D + chunk * 8) =
            make_uint2(h[0] | (h[1] << 16), h[2] | (h[3] << 16));
      }
    }
  } else {
    // code = rint(fl(x * inv)): the product is rounded once (__fmul_rn), then adding 1.5 * 2^23
    // rounds it to the nearest integer, ties to even (float32 spacing is 1 on [2^23, 2^24)), and the
    // low byte of the sum's bit pattern is the code in two's complement.  No clamp is needed:
    // |x| <= amax and inv <= (127/amax)(1 + 2^-24), so |fl(x * inv)| < 127.5 and |code| <= 127.
    // (A zero block has inv = 0 and gives code 0.)
#pragma unroll
    for (int ps = 0; ps < PASSES; ++ps) {
      const int row = ps * RPP + r_in;
      if (row < cnt) {
        uint32_t b[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) b[c] = __float_as_uint(__fadd_rn(__fmul_rn(x[ps][c], inv), 12582912.0f));
        const uint32_t w0 = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
        const uint32_t w1 = __byte_perm(__byte_perm(b[4], b[5], 0x0040), __byte_perm(b[6], b[7], 0x0040), 0x5410);
        *reinterpret_cast<uint2*>(dst + (size_t)row * D + chunk * 8) = make_uint2(w0, w1);
      }
    }
  }
}

}  // namespace tattn
