#pragma once
// decode_launch.cuh - host side of the KV-cache decode path: split count, workspace layout, TMA
// descriptors and the two launches (split kernel, then the log-sum-exp merge when there is more
// than one split).  Included by api.cu inside its anonymous namespace (after tma_host.cuh).

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

// Splits of each sequence's key range.  Requested > 0: that many (at most one per key tile).
// 0: enough CTAs to give every SM one (batch, kv head, split), keeping at least 4 key tiles of
// 128 per split so that each CTA's TMA ring reaches steady state.
int decode_splits(int B, int Hkv, int Nk, int requested) {
  const int tiles = (Nk + 127) / 128;
  if (requested > 0) return std::min(requested, tiles);
  const long long units = (long long)B * Hkv;
  long long s = device_sm_count() / units;
  s = std::min<long long>(s, std::max(1, tiles / 4));
  return (int)std::max<long long>(1, s);
}

struct DecWs {
  size_t part_o, part_lse, total;
};

DecWs decode_ws(int B, int Hq, int Nq, int nsplit) {
  DecWs w{};
  if (nsplit <= 1) return w;
  const size_t rows = (size_t)B * Hq * Nq;
  w.part_o = 0;
  w.part_lse = align256((size_t)nsplit * rows * 128 * sizeof(float));
  w.total = w.part_lse + align256((size_t)nsplit * rows * sizeof(float));
  return w;
}

template <int RP, bool FP16>
int launch_decode_t(const void* q, const void* k, const void* v, const DecParams& p, cudaStream_t stream) {
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
  const long long grid = (long long)p.B * p.Hkv * p.nsplit;
  kern<<<(unsigned)grid, C::kThreads, C::SMEM_BYTES, stream>>>(tq, tk, tv, p);
  TATTN_CUDA(cudaGetLastError());
  if (p.nsplit > 1) {
    const int rows = p.B * p.Hq * p.Nq;
    attn_decode_combine_kernel<FP16><<<(unsigned)rows, 128, 0, stream>>>(p.part_o, p.part_lse, p.nsplit, rows, p.o,
                                                                         p.lse);
    TATTN_CUDA(cudaGetLastError());
  }
  return ATTN_OK;
}

int launch_decode(const void* q, const void* k, const void* v, int dtype, const DecParams& p, cudaStream_t stream) {
  const bool fp16 = dtype == ATTN_FP16;
  switch (decode_rp(p.R)) {
    case 16: return fp16 ? launch_decode_t<16, true>(q, k, v, p, stream) : launch_decode_t<16, false>(q, k, v, p, stream);
    case 32: return fp16 ? launch_decode_t<32, true>(q, k, v, p, stream) : launch_decode_t<32, false>(q, k, v, p, stream);
    case 64: return fp16 ? launch_decode_t<64, true>(q, k, v, p, stream) : launch_decode_t<64, false>(q, k, v, p, stream);
    default: return ATTN_ERR_UNSUPPORTED;
  }
}

// Argument checks shared by attn_decode and attn_decode_workspace_bytes.
int check_decode_shape(int B, int Hq, int Hkv, int Nq, int Nk, int d, int num_splits) {
  if (B < 1 || Hq < 1 || Hkv < 1 || Nq < 1 || Nk < 1 || num_splits < 0) return ATTN_ERR_ARG;
  if (Hq % Hkv || Nq > Nk) return ATTN_ERR_ARG;
  if (d != 128) return ATTN_ERR_UNSUPPORTED;
  if ((long long)(Hq / Hkv) * Nq > kDecodeMaxRows) return ATTN_ERR_UNSUPPORTED;
  if ((long long)B * Hkv > (1 << 24) || Nk > (1 << 30) || (long long)B * Hq * Nq > (1 << 30) || num_splits > 4096)
    return ATTN_ERR_UNSUPPORTED;
  return ATTN_OK;
}
