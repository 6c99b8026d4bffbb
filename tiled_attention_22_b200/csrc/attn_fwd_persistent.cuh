#pragma once
// attn_fwd_persistent.cuh - the fused attention forward kernel with persistent CTAs (one per SM),
// for sm_100a.  It computes what attn_fwd_kernel computes (same tiles, the same per-tile softmax,
// Q K^T and P V code, the same epilogue; attn_fwd_kernels.cuh describes the method and its
// sources), but a CTA runs many work items instead of one, so the per-CTA costs (launch, barrier
// set-up, TMEM allocation, the first Q and K loads, the wait for the last tile's epilogue) are paid
// once per SM and the next item's first loads and Q K^T overlap the previous item's end.  Used
// for 16-bit Q K^T at d = 128, where it measured 3-6% faster on the named workloads; the 8-bit
// modes and d = 64 measured no gain and keep one CTA per item (attn_fwd_kernel).
#include "attn_fwd_kernels.cuh"

namespace tattn {

// Roles beyond those of attn_fwd_kernel: warp 10 loads Q, warp 11 hands out work items; an item
// slot is released by the 8 softmax warps and the K/V, MMA and Q warps.
constexpr int kFwdQWarp = 10;
constexpr int kFwdSchedWarp = 11;
constexpr int kFwdItemConsumers = 8 + 3;
enum : int { W_ITEM = 0x70 };

// Shared-memory layout: attn_fwd_kernel's tiles and O staging, then the barriers
//   q_full[2] q_empty[2] k_full[KS] k_empty[KS] v_full[VS] v_empty[VS] s_full[2] p_full[2]
//   o_done[2] drain claim item_full[4] item_empty[4]
// then 4 item slots (idx, mb, kvz, bh, n0, n1), the TMEM slot and the abort flag.
template <int D, bool BYTE>
struct FwdPersistCfg : FwdCfg<D, BYTE> {
  using Base = FwdCfg<D, BYTE>;
  static_assert(!Base::PSMEM, "the persistent kernel keeps P in tensor memory");
  static constexpr int ITEM_RING = 4;
  static constexpr int ITEM_INTS = 6;
  static constexpr int NBAR = 4 + 2 * Base::KSTAGES + 2 * Base::VSTAGES + 6 + 2 + 2 * ITEM_RING;
  static constexpr int SMEM_USED = Base::OFF_BAR + NBAR * 8 + ITEM_RING * ITEM_INTS * 4 + 32;
  static constexpr int SMEM_BYTES = (SMEM_USED + 1024) > 120 * 1024 ? (SMEM_USED + 1024) : 120 * 1024;
  static_assert(SMEM_USED + 1024 <= 232448, "shared memory budget");
};

// One work item: query rows [kItemRows mb, kItemRows (mb + 1)) of query head bh, reading kv head kvz; n0 and n1
// key tiles for its two 128-row query tiles (0 for a tile past N).
struct FwdItem {
  int mb, kvz, bh, n0, n1;
};

// Items are ordered in sections of sec_kv consecutive (batch, kv head) pairs, sized on the host so
// that a section's K and V fit comfortably in L2: all query heads and m blocks of a section run
// close together and share those K/V tiles through L2.  Inside a section, m blocks go heaviest
// first under causal masking (longest rows start first), query heads fastest: the order in which
// attn_fwd_kernel's CTAs are numbered.
__device__ __forceinline__ FwdItem fwd_item(const FwdParams& p, int idx) {
  const int G = p.Hq / p.Hkv;
  const int n_bkv = p.B * p.Hkv;
  const int per_sec = p.sec_kv * G * p.n_mblocks;
  const int sec = idx / per_sec;
  const int kv0 = sec * p.sec_kv;
  const int nkv_sec = min(p.sec_kv, n_bkv - kv0);
  const int rr = idx - sec * per_sec;
  const int mb_rank = rr / (nkv_sec * G);
  const int within = rr - mb_rank * (nkv_sec * G);
  FwdItem it;
  it.kvz = kv0 + within / G;  // b * Hkv + kv head
  it.mb = p.causal ? p.n_mblocks - 1 - mb_rank : mb_rank;
  const int b = it.kvz / p.Hkv;
  const int h = (it.kvz - b * p.Hkv) * G + within % G;
  it.bh = b * p.Hq + h;
  const int nkv = (p.Nk + 127) / 128;
  auto key_tiles = [&](int t) {
    const int row0 = it.mb * kItemRows + 128 * t;
    if (row0 >= p.N || (TATTN_QT1 && t == 1)) return 0;
    return p.causal ? min(nkv, row0 / 128 + 1) : nkv;
  };
  it.n0 = key_tiles(0);
  it.n1 = key_tiles(1);
  return it;
}

// Persistent CTAs (one per SM): warp 11 takes work items from a global ticket counter (cleared
// before the launch) and hands them, decoded, to the other roles through a ring of ITEM_RING
// shared-memory slots, so items go to CTAs in order, as they free up, and one CTA's set-up, TMEM
// allocation and first loads serve many items.  Across items the roles keep their ring positions
// and barrier phases; the next item's Q is loaded (warp 10) as soon as the MMAs of the previous
// item no longer read that query tile's buffer, and its first Q K^T is issued right after the
// previous item's last P V, while the softmax warps still write out the previous O.
template <int D, int QK, bool FP16>
__global__ void __launch_bounds__(FwdRoles<false>::kThreads, 1)
    attn_fwd_persistent_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                               const FwdParams p, int n_items, unsigned* tickets) {
  constexpr bool QUANT = QK != QK_F16;  // 8-bit codes with per-block scales sq, sk and the lse bias
  using C = FwdPersistCfg<D, QUANT>;
  using R = FwdRoles<false>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* q_empty = q_full + 2;
  uint64_t* k_full = q_empty + 2;
  uint64_t* k_empty = k_full + C::KSTAGES;
  uint64_t* v_full = k_empty + C::KSTAGES;
  uint64_t* v_empty = v_full + C::VSTAGES;
  uint64_t* s_full = v_empty + C::VSTAGES;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_done = p_full + 2;
  uint64_t* drain = o_done + 2;
  uint64_t* claim = drain + 1;  // the K/V loads of an item are all issued: take the next item
  uint64_t* item_full = claim + 1;
  uint64_t* item_empty = item_full + C::ITEM_RING;
  volatile int* item_slot = reinterpret_cast<volatile int*>(item_empty + C::ITEM_RING);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(const_cast<int*>(item_slot) + C::ITEM_RING * C::ITEM_INTS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], TATTN_PFULL_PER_WARP ? R::kThreadsPerTile / 32 : R::kThreadsPerTile);
      mbar_init(&o_done[i], 1);
    }
    for (int i = 0; i < C::KSTAGES; ++i) { mbar_init(&k_full[i], 1); mbar_init(&k_empty[i], 1); }
    for (int i = 0; i < C::VSTAGES; ++i) { mbar_init(&v_full[i], 1); mbar_init(&v_empty[i], 1); }
    for (int i = 0; i < C::ITEM_RING; ++i) { mbar_init(&item_full[i], 1); mbar_init(&item_empty[i], kFwdItemConsumers); }
    mbar_init(drain, 1);
    mbar_init(claim, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == R::kMmaWarp) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == R::kTmaWarp && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmO);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Item k of this CTA, decoded by the work-item warp (all lanes of the calling warp wait; lane 0
  // releases the slot).  Returns false on abort; it.bh < 0: no more items.
  auto take_item = [&](int k, FwdItem& it) -> bool {
    const int s = k % C::ITEM_RING;
    const bool waited = mbar_wait(&item_full[s], (k / C::ITEM_RING) & 1, abort_flag, W_ITEM + 1);
    if (!__all_sync(0xffffffffu, waited)) return false;
    const volatile int* f = item_slot + s * C::ITEM_INTS;
    it.mb = f[1];
    it.kvz = f[2];
    it.bh = f[3];
    it.n0 = f[4];
    it.n1 = f[5];
    if (f[0] < 0) it.bh = -1;
    __syncwarp();
    if (lane == 0) mbar_arrive(&item_empty[s]);
    return true;
  };
  const int nkv = (p.Nk + 127) / 128;

  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sV = smem + C::OFF_V;

  if (warp >= R::kSoftmaxWarps) {
    regs_decrease<R::kRegsProducer>();
  if (warp == kFwdSchedWarp) {
    // ================================ work items ================================
    // An item is taken from the ticket counter only when the K/V loads of the previous one are
    // all issued (a few key tiles before that item ends), so a CTA never holds work that another
    // CTA could start sooner.
    if (lane == 0) {
      for (int k = 0;; ++k) {
        const int s = k % C::ITEM_RING;
        if (!mbar_wait(&item_empty[s], ((k / C::ITEM_RING) & 1) ^ 1, abort_flag, W_ITEM + 2)) break;
        if (k > 0 && !mbar_wait(claim, (k - 1) & 1, abort_flag, W_ITEM + 3)) break;
        const unsigned tk = atomicAdd(tickets, 1u);
        const int idx = tk < (unsigned)n_items ? (int)tk : -1;
        volatile int* f = item_slot + s * C::ITEM_INTS;
        f[0] = idx;
        if (idx >= 0) {
          const FwdItem it = fwd_item(p, idx);
          f[1] = it.mb;
          f[2] = it.kvz;
          f[3] = it.bh;
          f[4] = it.n0;
          f[5] = it.n1;
        }
        mbar_arrive(&item_full[s]);  // release: the slot is written before the phase completes
        if (idx < 0) break;
      }
    }
    __syncwarp();
  } else if (warp == kFwdQWarp) {
    // ================================ Q loads ================================
    bool ok = true;
    int qc[2] = {0, 0};  // Q tiles loaded per query tile
    for (int k = 0; ok; ++k) {
      FwdItem it;
      if (!(ok = take_item(k, it)) || it.bh < 0) break;
      if (lane == 0) {
        // start the item's Q on its way to L2 now; the copy into shared memory waits for the buffer
        for (int t = 0; t < 2; ++t)
          if ((t ? it.n1 : it.n0) > 0)
            for (int pn = 0; pn < C::QK_PANELS; ++pn)
              tma_prefetch_l2_3d(&tmQ, pn * C::QK_BOX_X, it.mb * kItemRows + 128 * t, it.bh);
        const uint64_t pol_stream = policy_evict_first();
        for (int t = 0; t < 2 && ok; ++t) {
          if ((t ? it.n1 : it.n0) == 0) continue;
          // the previous item's Q K^T products with this buffer have completed
          if (!(ok = mbar_wait(&q_empty[t], (qc[t] & 1) ^ 1, abort_flag, W_LOAD + 3))) break;
          mbar_arrive_expect_tx(&q_full[t], C::Q_TILE);
          for (int pn = 0; pn < C::QK_PANELS; ++pn)
            tma_load_3d(sQ + t * C::Q_TILE + pn * C::QK_PANEL_BYTES, &tmQ, pn * C::QK_BOX_X, it.mb * kItemRows + 128 * t,
                        it.bh, &q_full[t], pol_stream);
          ++qc[t];
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
    }
    if (!ok && lane == 0) {
      // Drain: only the last Q load of each tile can still be in flight.
      for (int t = 0; t < 2; ++t)
        if (qc[t] > 0) mbar_wait(&q_full[t], (qc[t] - 1) & 1, nullptr, W_DRAIN + 1, 200000000ull);
    }
    __syncwarp();
  } else if (warp == R::kTmaWarp) {
    // ================================ K and V loads ================================
    bool ok = true;
    int g = 0;  // ring position: key tiles loaded so far, over all items
    int k_issued = 0, v_issued = 0;
    for (int k = 0; ok; ++k) {
      FwdItem it;
      if (!(ok = take_item(k, it)) || it.bh < 0) break;
      const int nmax = max(it.n0, it.n1);
      if (lane == 0) {
        const uint64_t pol_keep = policy_evict_last();
        for (int j = 0; j < nmax && ok; ++j) {
          const int gj = g + j;
          const int ks = gj % C::KSTAGES, vs = gj % C::VSTAGES;
          if (!(ok = mbar_wait(&k_empty[ks], ((gj / C::KSTAGES) & 1) ^ 1, abort_flag, W_LOAD + 1))) break;
          mbar_arrive_expect_tx(&k_full[ks], C::K_TILE);
          for (int pn = 0; pn < C::QK_PANELS; ++pn)
            tma_load_3d(sK + ks * C::K_TILE + pn * C::QK_PANEL_BYTES, &tmK, pn * C::QK_BOX_X, j * 128, it.kvz,
                        &k_full[ks], pol_keep);
          k_issued = gj + 1;
          if (!(ok = mbar_wait(&v_empty[vs], ((gj / C::VSTAGES) & 1) ^ 1, abort_flag, W_LOAD + 2))) break;
          mbar_arrive_expect_tx(&v_full[vs], C::V_TILE);
          for (int pn = 0; pn < C::V_PANELS; ++pn)
            tma_load_3d(sV + vs * C::V_TILE + pn * C::V_PANEL_BYTES, &tmV, pn * 64, j * 128, it.kvz, &v_full[vs],
                        pol_keep);
          v_issued = gj + 1;
        }
        if (ok) mbar_arrive(claim);  // all of this item's loads are issued
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      g += nmax;
    }
    if (!ok && lane == 0) {
      // Drain: every issued copy must land before the CTA's shared memory is released.
      for (int j = max(0, k_issued - C::KSTAGES); j < k_issued; ++j)
        mbar_wait(&k_full[j % C::KSTAGES], (j / C::KSTAGES) & 1, nullptr, W_DRAIN + 2, 200000000ull);
      for (int j = max(0, v_issued - C::VSTAGES); j < v_issued; ++j)
        mbar_wait(&v_full[j % C::VSTAGES], (j / C::VSTAGES) & 1, nullptr, W_DRAIN + 3, 200000000ull);
    }
    __syncwarp();
  } else if (warp == R::kMmaWarp) {
    // ================================ MMA issuer ================================
    bool ok = true;
    int g = 0;                 // ring position of the item's first key tile
    int qm[2] = {0, 0};        // Q tiles consumed per query tile
    int pc[2] = {0, 0};        // P tiles consumed per query tile
    const uint32_t q_addr = smem_u32(sQ), k_addr = smem_u32(sK), v_addr = smem_u32(sV);
    for (int k = 0; ok; ++k) {
      FwdItem it;
      if (!(ok = take_item(k, it)) || it.bh < 0) break;
      const int n0 = it.n0, n1 = it.n1, nmax = max(n0, n1);
      if (lane == 0) {
        auto n_of = [&](int t) { return t ? n1 : n0; };
        auto users_first = [&](int j) { return j < n0 ? 0 : 1; };
        auto users_last = [&](int j) { return j < n1 ? 1 : 0; };
        // prologue: S_t(0) for both tiles
        if (nmax > 0) {
          ok = mbar_wait(&k_full[g % C::KSTAGES], (g / C::KSTAGES) & 1, abort_flag, W_MMA + 1);
          for (int t = 0; t < 2 && ok; ++t) {
            if (n_of(t) == 0) continue;
            if (!(ok = mbar_wait(&q_full[t], qm[t] & 1, abort_flag, W_MMA + 2))) break;
            ++qm[t];
            tc_fence_after();
            issue_qk<D, QK, FP16>(tmem + C::tm_s(t), q_addr + t * C::Q_TILE, k_addr + (g % C::KSTAGES) * C::K_TILE);
            mma_commit(&s_full[t]);
            if (n_of(t) == 1) mma_commit(&q_empty[t]);  // the tile's last Q K^T of this item
            if (users_last(0) == t) mma_commit(&k_empty[g % C::KSTAGES]);
          }
        }
        for (int j = 0; j < nmax && ok; ++j) {
          const int vs = (g + j) % C::VSTAGES;
          const int ks1 = (g + j + 1) % C::KSTAGES;
          for (int t = 0; t < 2 && ok; ++t) {
            if (j >= n_of(t)) continue;
            // V(j) and K(j + 1) first (normally loaded long before), then P
            if (users_first(j) == t)
              if (!(ok = mbar_wait(&v_full[vs], ((g + j) / C::VSTAGES) & 1, abort_flag, W_MMA + 4))) break;
            if (j + 1 < n_of(t) && users_first(j + 1) == t)
              if (!(ok = mbar_wait(&k_full[ks1], ((g + j + 1) / C::KSTAGES) & 1, abort_flag, W_MMA + 5))) break;
            if (!(ok = mbar_wait(&p_full[t], pc[t] & 1, abort_flag, W_MMA + 3))) break;
            ++pc[t];
            tc_fence_after();
            issue_pv<D, FP16>(tmem + C::tm_o(t), tmem + C::tm_s(t), v_addr + vs * C::V_TILE, j > 0);
            if (j + 1 == n_of(t)) mma_commit(&o_done[t]);  // the tile's last P V: O is final
            if (users_last(j) == t) mma_commit(&v_empty[vs]);
            if (j + 1 < n_of(t)) {
              issue_qk<D, QK, FP16>(tmem + C::tm_s(t), q_addr + t * C::Q_TILE, k_addr + ks1 * C::K_TILE);
              mma_commit(&s_full[t]);
              if (j + 2 == n_of(t)) mma_commit(&q_empty[t]);  // the tile's last Q K^T of this item
              if (users_last(j + 1) == t) mma_commit(&k_empty[ks1]);
            }
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      g += nmax;
    }
    if (!ok && lane == 0) {
      // Drain: wait until every MMA issued so far has completed before TMEM is released.
      mma_commit(drain);
      mbar_wait(drain, 0, nullptr, W_DRAIN + 4, 200000000ull);
    }
    __syncwarp();
  }  // (no other producer warps)
  } else {
    regs_increase<R::kRegsSoftmax>();
    // ================================ softmax (one row per thread) ================================
    const int t = warp >> 2, wq = warp & 3;
    const uint32_t tS = tmem + C::tm_s(t) + ((uint32_t)(wq * 32) << 16);
    const uint32_t tO = tmem + C::tm_o(t) + ((uint32_t)(wq * 32) << 16);
    const int nblk = (p.N + 127) / 128;
    uint8_t* slot = smem + C::OFF_O + warp * C::O_SLOT;
    bool ok = true;
    int sc_cnt = 0;  // S tiles of this query tile consumed over all items (s_full phase)
    int oc_cnt = 0;  // items with a non-empty tile t (o_done phase)
    for (int k = 0; ok; ++k) {
      FwdItem it;
      if (!(ok = take_item(k, it)) || it.bh < 0) break;
      const int nt = t ? it.n1 : it.n0;
      const int row0 = it.mb * kItemRows + 128 * t;
      const int row = row0 + wq * 32 + lane;
      const int bh = it.bh;
      // (an empty tile, row0 >= N, reads nothing: its sq entry does not exist)
      const float sq_scale = (QUANT && nt > 0) ? p.sq[(size_t)bh * nblk + row0 / 128] * p.scale_log2 : p.scale_log2;
      float m_run = -INFINITY, l_run = 0.f;
      // 8-bit modes: the key block's scale, loaded one tile ahead so that its latency is off the
      // tile's critical path, and the row's lse bias, loaded now so that the epilogue does not
      // wait for it
      const float* skp = p.sk + (size_t)it.kvz * nkv;
      float sk_next = (QUANT && nt > 0) ? __ldg(skp) : 0.f;
      const float lse_bias = (QUANT && p.lse != nullptr && nt > 0 && row < p.N) ? __ldg(&p.bias[(size_t)bh * p.N + row]) : 0.f;
      for (int j = 0; j < nt; ++j) {
        float sk_j = 0.f;
        if constexpr (QUANT) {
          sk_j = sk_next;
          if (j + 1 < nt) sk_next = __ldg(skp + j + 1);
        }
        ok = mbar_wait(&s_full[t], (sc_cnt + j) & 1, abort_flag, W_SOFTMAX + 1);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        float sc = QUANT ? sq_scale * sk_j : sq_scale;
        if constexpr (QUANT) sc = fmaxf(sc, 1e-30f);  // a zero block: keep -inf * sc = -inf for masks
        // the causal diagonal tile (key > query) and the ragged last key tile (key >= Nk) are
        // masked; keys [0, lim) of the tile are visible
        const int col0 = j * 128;
        const bool diag = p.causal && (j == nt - 1);
        if (diag || (col0 + 128 > p.Nk)) {
          const int lim = (diag ? min(row + 1, p.Nk) : p.Nk) - col0;
          ok = softmax_step<D, QK, FP16, true>(tS, tO, sc, lim, j, m_run, l_run, &o_done[t], abort_flag);
        } else {
          ok = softmax_step<D, QK, FP16, false>(tS, tO, sc, 128, j, m_run, l_run, &o_done[t], abort_flag);
        }
        if (!ok) break;
        tmem_st_wait();
        tc_fence_before();
        if (TATTN_PFULL_PER_WARP) {
          // one arrival per warp: every lane's TMEM stores are complete (wait::st) and fenced
          // before the warp synchronises; lane 0 then releases them to the MMA thread
          __syncwarp();
          if (lane == 0) mbar_arrive(&p_full[t]);
        } else {
          mbar_arrive(&p_full[t]);
        }
      }
      if (!ok) break;
      sc_cnt += nt;
      if (nt > 0) {
        ok = mbar_wait(&o_done[t], oc_cnt & 1, abort_flag, W_SOFTMAX + 3);
        ok = __all_sync(0xffffffffu, ok);
        ++oc_cnt;
        if (!ok) break;
        tc_fence_after();
        const float inv_l = 1.0f / l_run;
        // O through this warp's shared-memory slot, one 64-column panel at a time, each panel
        // written to global memory by one TMA store of the warp's 32 rows (rows past N are
        // clipped by the tensor map).  Slot layout: row r at r * 128 bytes, 16-byte chunk c at
        // position c ^ (r & 7) (the 128-byte swizzle of the tensor map).
        const uint32_t swz = (uint32_t)(lane & 7);
        const int y0 = row0 + wq * 32;
#pragma unroll
        for (int pn = 0; pn < D / 64; ++pn) {
          // the slot's previous store (earlier panel or item) has finished reading it
          if (lane == 0) bulk_wait_group_read0();
          __syncwarp();
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            uint32_t o[32];
            tmem_ld32(tO + 64 * pn + 32 * cc, o);
            tmem_ld_wait(o);
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pk[i] = pack2(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l, FP16);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              *reinterpret_cast<uint4*>(slot + lane * 128 + (((uint32_t)(cc * 4 + v) ^ swz) << 4)) =
                  make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
          }
          fence_async_smem();  // the slot's generic stores before the TMA engine reads it
          __syncwarp();
          if (lane == 0 && y0 < p.N) {
            tma_store_3d(&tmO, slot, pn * 64, y0, bh);
            bulk_commit_group();
          }
        }
        if (p.lse != nullptr && row < p.N) {
          float lse = (m_run + __log2f(l_run)) * 0.69314718055994531f;
          if constexpr (QUANT) lse += lse_bias;
          p.lse[(size_t)bh * p.N + row] = lse;
        }
      }
    }
    if (!ok) {
      // make sure this thread's TMEM traffic is finished before teardown
      tmem_st_wait();
    }
    // the slot must stay until the last store has read it
    if (lane == 0) bulk_wait_group_read0();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == R::kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace tattn
