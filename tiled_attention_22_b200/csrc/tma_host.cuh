#pragma once
// tma_host.cuh - host-side TMA tensor maps: a [B, H, N, d] tensor viewed as (d, N, B*H) so that
// rows past N of one head read as zeros.  Included by api.cu inside its anonymous namespace.
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// [BH, N, d] view of a [B, H, N, d] tensor; box = box_x elements x box_y rows x 1 head.
int make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem_bytes, int d, int N, int BH,
             int box_x, CUtensorMapSwizzle swz, int box_y = 128) {
  auto fn = encode_fn();
  if (!fn) {
    std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "cuTensorMapEncodeTiled unavailable");
    return ATTN_ERR_LAUNCH;
  }
  // The encoder is a driver call and needs the device's context current on this thread.  A host
  // thread that has made no runtime call needing a context yet (a new thread whose streams came
  // from a pool) has none; cudaSetDevice on the current device makes its primary context current.
  int dev = 0;
  TATTN_CUDA(cudaGetDevice(&dev));
  TATTN_CUDA(cudaSetDevice(dev));
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)d * elem_bytes, (cuuint64_t)N * d * elem_bytes};
  cuuint32_t box[3] = {(cuuint32_t)box_x, (cuuint32_t)box_y, 1u};
  cuuint32_t estr[3] = {1u, 1u, 1u};
  CUresult r = fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return ATTN_ERR_LAUNCH;
  }
  return ATTN_OK;
}

CUtensorMapSwizzle swizzle_for(int row_bytes) {
  return row_bytes >= 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
}

