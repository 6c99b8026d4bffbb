// merge_kernels.cuh - the lse merge of partial attention results, for sm_100a.
//
// The "FlashAttention" glossary (aiunderstanding.org, deep-dive section and FAQ) computes softmax
// over key blocks with running maxima and sums and rescales the partial results; the same identity
// joins two results computed over disjoint key sets.  With O_a = softmax over keys A applied to V_A,
// lse_a = ln sum_{j in A} exp(s_j) (and the same for B):
//     lse = ln(exp(lse_a) + exp(lse_b)),   O = exp(lse_a - lse) O_a + exp(lse_b - lse) O_b.
// The APB article ("在长文本上比Flash Attention快10倍！…", section on the baselines) names ring
// attention as the exact sequence-parallel method: every device keeps its query block and the key/value
// blocks travel round a ring, each step's partial result merged in this way.
//
// HBM-bound: one warp per row, the fp32 accumulator read and written once, the 16-bit part read once.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

namespace tattn {

template <bool FP16>
__device__ __forceinline__ float half_to_float(uint16_t b) {
  if constexpr (FP16)
    return __half2float(__ushort_as_half(b));
  else
    return __uint_as_float((uint32_t)b << 16);
}

template <bool FP16>
__device__ __forceinline__ uint16_t float_to_half(float x) {
  if constexpr (FP16)
    return __half_as_ushort(__float2half_rn(x));
  else
    return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

// Per row r (rows = B*Hq*Nq, each d values):
//   first:  acc = part (the running result starts as the first partial result);
//   part == nullptr: acc unchanged (finalise only);
//   else:   acc = merge(acc, part) by the identity above, computed in float32.
//   out != nullptr: out[r] = acc converted to 16-bit (round to nearest even).
// A row whose lse is -inf has no keys; its O is 0 and it carries no weight.
template <int D, bool FP16>
__global__ void __launch_bounds__(256) lse_merge_kernel(float* __restrict__ o_acc, float* __restrict__ lse_acc,
                                                        const uint16_t* __restrict__ o_part,
                                                        const float* __restrict__ lse_part,
                                                        uint16_t* __restrict__ out, long long rows, int first) {
  constexpr int PER = D / 32;  // values per lane (4 for d = 128, 2 for d = 64)
  const int lane = threadIdx.x & 31;
  const long long warps = (long long)gridDim.x * (blockDim.x / 32);
  for (long long r = (long long)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32; r < rows; r += warps) {
    float* acc = o_acc + r * D + lane * PER;
    float o[PER];
    float l;
    if (o_part != nullptr) {
      const uint16_t* part = o_part + r * D + lane * PER;
      float p[PER];
      if constexpr (PER == 4) {
        const uint2 raw = *reinterpret_cast<const uint2*>(part);
        p[0] = half_to_float<FP16>(raw.x & 0xffffu);
        p[1] = half_to_float<FP16>(raw.x >> 16);
        p[2] = half_to_float<FP16>(raw.y & 0xffffu);
        p[3] = half_to_float<FP16>(raw.y >> 16);
      } else {
        const uint32_t raw = *reinterpret_cast<const uint32_t*>(part);
        p[0] = half_to_float<FP16>(raw & 0xffffu);
        p[1] = half_to_float<FP16>(raw >> 16);
      }
      const float lp = lse_part[r];
      if (first) {
#pragma unroll
        for (int i = 0; i < PER; ++i) o[i] = p[i];
        l = lp;
      } else {
        const float la = lse_acc[r];
        float a[PER];
        if constexpr (PER == 4) {
          const float4 v = *reinterpret_cast<const float4*>(acc);
          a[0] = v.x; a[1] = v.y; a[2] = v.z; a[3] = v.w;
        } else {
          const float2 v = *reinterpret_cast<const float2*>(acc);
          a[0] = v.x; a[1] = v.y;
        }
        const float m = fmaxf(la, lp);
        if (m == -INFINITY) {  // neither part has a key
#pragma unroll
          for (int i = 0; i < PER; ++i) o[i] = 0.f;
          l = -INFINITY;
        } else {
          const float wa = expf(la - m), wp = expf(lp - m);  // one of them is 1
          const float s = wa + wp;
          const float ia = wa / s, ip = wp / s;
#pragma unroll
          for (int i = 0; i < PER; ++i) o[i] = fmaf(ia, a[i], ip * p[i]);
          l = m + logf(s);
        }
      }
      if constexpr (PER == 4)
        *reinterpret_cast<float4*>(acc) = make_float4(o[0], o[1], o[2], o[3]);
      else
        *reinterpret_cast<float2*>(acc) = make_float2(o[0], o[1]);
      if (lane == 0) lse_acc[r] = l;
    } else {
      if constexpr (PER == 4) {
        const float4 v = *reinterpret_cast<const float4*>(acc);
        o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
      } else {
        const float2 v = *reinterpret_cast<const float2*>(acc);
        o[0] = v.x; o[1] = v.y;
      }
    }
    if (out != nullptr) {
      uint16_t* dst = out + r * D + lane * PER;
      if constexpr (PER == 4)
        *reinterpret_cast<uint2*>(dst) = make_uint2(float_to_half<FP16>(o[0]) | ((uint32_t)float_to_half<FP16>(o[1]) << 16),
                                                    float_to_half<FP16>(o[2]) | ((uint32_t)float_to_half<FP16>(o[3]) << 16));
      else
        *reinterpret_cast<uint32_t*>(dst) = float_to_half<FP16>(o[0]) | ((uint32_t)float_to_half<FP16>(o[1]) << 16);
    }
  }
}

}  // namespace tattn
