#pragma once
// attn_fwd_launch.cuh - host-side launch of the fused attention kernel: TMA descriptors for Q, K, V
// and O, one-time per-device kernel setup (shared memory size, register-split check), the choice
// between one CTA per work item and persistent CTAs, and the grid.  Included by api.cu inside its
// anonymous namespace (after cuda_fail / TATTN_CUDA and device_sm_count).
#ifndef TATTN_SPLIT
#define TATTN_SPLIT 0
#endif

// Persistent launches take their work items from a ticket counter that no other launch may touch
// while they run; the counter is cleared on the launch's stream just before the kernel.  Counters
// live in the library, kTicketSlots per device, one per stream, keyed by the stream's id
// (cudaStreamGetId: unique in the process for the life of the program).  The id, unlike the handle
// value, tells apart streams that share a handle: cudaStreamPerThread names a different stream in
// each host thread, and a destroyed stream's handle value can come back for a new stream.  Launches
// from streams past the kTicketSlots-th use one CTA per item instead (the same results).
//
// A launch recorded by stream capture would carry its counter's address into every replay of the
// graph, on whatever stream the replay runs, alongside direct calls on the capturing stream; so a
// capturing stream gets no counter and the launch uses one CTA per item.
constexpr int kTicketSlots = 256;
__device__ unsigned g_fwd_tickets[kTicketSlots];

unsigned* fwd_ticket_counter(cudaStream_t stream) {
  static std::mutex mu;
  static unsigned* base[kMaxDevices];
  static unsigned long long owner[kMaxDevices][kTicketSlots];
  static int used[kMaxDevices];
  cudaStreamCaptureStatus capture = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &capture) != cudaSuccess || capture != cudaStreamCaptureStatusNone) {
    cudaGetLastError();
    return nullptr;
  }
  unsigned long long id = 0;
  if (cudaStreamGetId(stream, &id) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (base[dev] == nullptr) {
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_fwd_tickets) != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    base[dev] = static_cast<unsigned*>(addr);
  }
  for (int i = 0; i < used[dev]; ++i)
    if (owner[dev][i] == id) return base[dev] + i;
  if (used[dev] == kTicketSlots) return nullptr;
  owner[dev][used[dev]] = id;
  return base[dev] + used[dev]++;
}

// Once per device and kernel: allow the dynamic shared memory, and check the register split.  The
// kernels move registers between warpgroups with setmaxnreg; the increase only completes if the
// registers the CTA is launched with cover the split, so refuse to launch otherwise.
template <class Kern>
int setup_fwd_kernel(Kern kern, int smem_bytes, std::atomic<int>* checked) {
  using R = FwdRoles<TATTN_SPLIT != 0>;
  int dev = 0;
  TATTN_CUDA(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return ATTN_ERR_LAUNCH;
  if (checked[dev].load(std::memory_order_acquire) != 1) {
    TATTN_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes));
    cudaFuncAttributes attr;
    TATTN_CUDA(cudaFuncGetAttributes(&attr, kern));
    if ((long long)attr.numRegs * R::kThreads <
            128LL * (R::kSoftmaxWarps / 4 * R::kRegsSoftmax + R::kRegsProducer) ||
        attr.maxThreadsPerBlock < R::kThreads) {
      std::snprintf(g_last_cuda_error, sizeof(g_last_cuda_error),
                    "fused kernel built with %d registers/thread: too few for its register split", attr.numRegs);
      return ATTN_ERR_LAUNCH;
    }
    checked[dev].store(1, std::memory_order_release);
  }
  return ATTN_OK;
}

template <int D, int QK, bool FP16>
int launch_fwd_t(const void* q, const void* k, const void* v, const FwdParams& p, cudaStream_t stream) {
  constexpr bool BYTE = QK != QK_F16;
  using C = FwdCfg<D, BYTE>;
  constexpr bool SPLIT = TATTN_SPLIT != 0;
  using R = FwdRoles<SPLIT>;
  CUtensorMap tq, tk, tv, to;
  const CUtensorMapDataType qk_dt =
      BYTE ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : (FP16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
  const CUtensorMapDataType v_dt = FP16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  int rc;
  if ((rc = make_map(&tq, q, qk_dt, C::QK_ELEM, D, p.N, p.B * p.Hq, C::QK_BOX_X, swizzle_for(C::QK_ROW)))) return rc;
  if ((rc = make_map(&tk, k, qk_dt, C::QK_ELEM, D, p.Nk, p.B * p.Hkv, C::QK_BOX_X, swizzle_for(C::QK_ROW)))) return rc;
  if ((rc = make_map(&tv, v, v_dt, 2, D, p.Nk, p.B * p.Hkv, 64, CU_TENSOR_MAP_SWIZZLE_128B))) return rc;
  // O: the epilogue's stores, 64 columns x 32 rows (one softmax warp's rows) per box
  if ((rc = make_map(&to, p.o, v_dt, 2, D, p.N, p.B * p.Hq, 64, CU_TENSOR_MAP_SWIZZLE_128B, 32))) return rc;
  const long long items = (long long)p.n_mblocks * p.B * p.Hq;
  // Persistent CTAs (one per SM) for 16-bit Q K^T at d = 128, where they measured 3-6% faster on
  // the named workloads (the 8-bit modes and d = 64 measured no gain); not under a row prefix mask
  // (its per-tile limits are read once per CTA) nor with the four-threads-per-row variant.
#ifndef TATTN_PERSIST_BYTE
#define TATTN_PERSIST_BYTE 0
#endif
  if constexpr ((QK == QK_F16 || TATTN_PERSIST_BYTE) && D == 128 && !SPLIT) {
    unsigned* tickets = p.row_lim == nullptr && items <= 0x7fffffffll ? fwd_ticket_counter(stream) : nullptr;
    if (tickets != nullptr) {
      using PC = FwdPersistCfg<D, BYTE>;
      auto pkern = attn_fwd_persistent_kernel<D, QK, FP16>;
      static std::atomic<int> checked_p[kMaxDevices];
      int rc2 = setup_fwd_kernel(pkern, PC::SMEM_BYTES, checked_p);
      if (rc2) return rc2;
      TATTN_CUDA(cudaMemsetAsync(tickets, 0, sizeof(unsigned), stream));
      const long long grid = std::min<long long>(items, device_sm_count());
      pkern<<<(unsigned)grid, R::kThreads, PC::SMEM_BYTES, stream>>>(tq, tk, tv, to, p, (int)items, tickets);
      TATTN_CUDA(cudaGetLastError());
      return ATTN_OK;
    }
  }
  auto kern = attn_fwd_kernel<D, QK, FP16, SPLIT>;
  static std::atomic<int> checked[kMaxDevices];
  if ((rc = setup_fwd_kernel(kern, C::SMEM_BYTES, checked))) return rc;
  const long long grid = items;
  kern<<<(unsigned)grid, R::kThreads, C::SMEM_BYTES, stream>>>(tq, tk, tv, to, p);
  TATTN_CUDA(cudaGetLastError());
  return ATTN_OK;
}

template <int QK>
int launch_fwd(const void* q, const void* k, const void* v, int d, int dtype, const FwdParams& p,
               cudaStream_t stream) {
  const bool fp16 = dtype == ATTN_FP16;
  if (d == 128) return fp16 ? launch_fwd_t<128, QK, true>(q, k, v, p, stream) : launch_fwd_t<128, QK, false>(q, k, v, p, stream);
  return fp16 ? launch_fwd_t<64, QK, true>(q, k, v, p, stream) : launch_fwd_t<64, QK, false>(q, k, v, p, stream);
}

FwdParams make_params(int B, int Hq, int Hkv, int N, int causal, float scale, void* o, float* lse, int Nk = -1,
                      const int* row_lim = nullptr) {
  FwdParams p{};
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.N = N;
  p.Nk = Nk < 0 ? N : Nk;
  p.row_lim = row_lim;
  p.causal = causal;
  p.n_mblocks = (N + kItemRows - 1) / kItemRows;
  // Scheduling sections: kv heads whose K and V (16-bit, d=128, the larger case) take at most
  // TATTN_L2_SECTION_MB (a quarter of the 126 MB L2 by default).
#ifndef TATTN_L2_SECTION_MB
#define TATTN_L2_SECTION_MB 32
#endif
  const long long kv_bytes = 2LL * p.Nk * 128 * 2;
  long long sec = ((long long)TATTN_L2_SECTION_MB << 20) / (kv_bytes > 0 ? kv_bytes : 1);
  if (sec < 1) sec = 1;
  if (sec > (long long)B * Hkv) sec = (long long)B * Hkv;
  p.sec_kv = (int)sec;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.o = o;
  p.lse = lse;
  return p;
}

