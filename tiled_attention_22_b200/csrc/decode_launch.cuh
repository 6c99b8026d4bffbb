#pragma once
// decode_launch.cuh - host side of the KV-cache decode path: CTA count, workspace layout, TMA
// descriptors and the launch of the persistent kernel (which also merges the pieces).  Included by api.cu inside its anonymous namespace (after tma_host.cuh).

// Query rows per kv head that the decode kernel takes: (Hq/Hkv) * Nq <= 64.
constexpr int kDecodeMaxRows = 64;

int decode_rp(int R) { return R <= 16 ? 16 : (R <= 32 ? 32 : (R <= kDecodeMaxRows ? 64 : 0)); }

int device_sm_count() {
  static std::atomic<int> cached[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return 148;
  }
  int n = cached[dev].load(std::memory_order_relaxed);
  if (n > 0) return n;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) {
    cudaGetLastError();
    n = 148;
  }
  cached[dev].store(n, std::memory_order_relaxed);
  return n;
}

// Persistent CTAs: requested > 0 takes that many, 0 one per SM; never more than there are key
// tiles in the largest possible problem (B * Hkv units of ceil(Nk / 128) tiles).
int decode_ctas(int B, int Hkv, int Nk, int requested) {
  const long long tiles = (long long)B * Hkv * ((Nk + 127) / 128);
  const long long want = requested > 0 ? requested : device_sm_count();
  return (int)std::max<long long>(1, std::min(want, tiles));
}

// Workspace: one arrival counter per unit (zero between calls), then the pieces' partial outputs
// and lse (slot = unit + CTA index, U + P - 1 slots).
struct DecWs {
  size_t part_o, part_lse, unit_arrived, total;
};

DecWs decode_ws(int B, int Hkv, int R, int P) {
  const size_t U = (size_t)B * Hkv, slots = U + (size_t)P - 1;
  DecWs w{};
  size_t off = 0;
  // the counters come first, so that their place does not depend on the CTA count and one
  // zeroed workspace serves calls with any count that fits
  w.unit_arrived = off; off += align256(U * sizeof(unsigned int));
  w.part_o = off;       off += align256(slots * R * 128 * sizeof(float));
  w.part_lse = off;     off += align256(slots * R * sizeof(float));
  w.total = off;
  return w;
}

template <int RP, bool FP16>
int launch_decode_t(const void* q, const void* k, const void* v, int ctas, const DecParams& p, cudaStream_t stream) {
  using C = DecCfg<RP>;
  const CUtensorMapDataType dt = FP16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  CUtensorMap tq, tk, tv;
  int rc;
  // Q: the R rows of one kv head's query group are contiguous ([B, Hq, Nq, d] with the group's
  // heads adjacent), so the view is (d, R, B*Hkv) and the box's rows past R read as zeros.
  if ((rc = make_map(&tq, q, dt, 2, 128, p.R, p.B * p.Hkv, 64, CU_TENSOR_MAP_SWIZZLE_128B, RP))) return rc;
  if ((rc = make_map(&tk, k, dt, 2, 128, p.Nk, p.B * p.Hkv, 64, CU_TENSOR_MAP_SWIZZLE_128B))) return rc;
  if ((rc = make_map(&tv, v, dt, 2, 128, p.Nk, p.B * p.Hkv, 64, CU_TENSOR_MAP_SWIZZLE_128B))) return rc;
  auto kern = attn_decode_kernel<RP, FP16>;
  static std::atomic<int> configured[kMaxDevices];
  int dev = 0;
  TATTN_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_LAUNCH;
  if (configured[dev].load(std::memory_order_acquire) != 1) {
    TATTN_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES));
    configured[dev].store(1, std::memory_order_release);
  }
  kern<<<(unsigned)ctas, C::kThreads, C::SMEM_BYTES, stream>>>(tq, tk, tv, p);
  TATTN_CUDA(cudaGetLastError());
  return ATTN_OK;
}

int launch_decode(const void* q, const void* k, const void* v, int dtype, int ctas, const DecParams& p,
                  cudaStream_t stream) {
  const bool fp16 = dtype == ATTN_FP16;
  switch (decode_rp(p.R)) {
    case 16:
      return fp16 ? launch_decode_t<16, true>(q, k, v, ctas, p, stream) : launch_decode_t<16, false>(q, k, v, ctas, p, stream);
    case 32:
      return fp16 ? launch_decode_t<32, true>(q, k, v, ctas, p, stream) : launch_decode_t<32, false>(q, k, v, ctas, p, stream);
    case 64:
      return fp16 ? launch_decode_t<64, true>(q, k, v, ctas, p, stream) : launch_decode_t<64, false>(q, k, v, ctas, p, stream);
    default: return ATTN_ERR_UNSUPPORTED;
  }
}

// Argument checks shared by attn_decode and attn_decode_workspace_bytes.
int check_decode_shape(int B, int Hq, int Hkv, int Nq, int Nk, int d, int num_ctas) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nk < 1 || num_ctas < 0) return ATTN_ERR_ARG;
  if (Hq % Hkv || Nq > Nk) return ATTN_ERR_ARG;
  if (d != 128) return ATTN_ERR_UNSUPPORTED;
  if ((long long)(Hq / Hkv) * Nq > kDecodeMaxRows) return ATTN_ERR_UNSUPPORTED;
  if ((long long)B * Hkv > (1 << 24) || Nk > (1 << 30) || (long long)B * Hq * Nq > (1 << 30) || num_ctas > 65536)
    return ATTN_ERR_UNSUPPORTED;
  return ATTN_OK;
}
