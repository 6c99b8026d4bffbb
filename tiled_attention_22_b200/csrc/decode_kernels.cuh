// decode_kernels.cuh - attention of a few new query tokens against a KV cache (decode / short-query
// forward), for sm_100a.
//
// What it computes: for every (batch b, query head h) and each of the Nq new tokens i,
// O = softmax(scale * q K^T [+ causal mask]) V over the first len_b cached keys of kv head
// h / (Hq/Hkv) ("注意力即一切：从 MHA 到 GQA", section 3.4: with a KV cache each new token's query
// attends to the stored keys and values of all earlier tokens; sections 2.2, 2.3 and 5.1 for the
// softmax, the mask and the head grouping).  The new tokens are the last Nq of the len_b, so under
// the causal mask token i sees keys 0 .. len_b - Nq + i.
//
// Why a second kernel: decoding reads the whole cache for a handful of query rows, so it is bound
// by HBM bandwidth, not by the tensor core.  The prefill kernel's 128-row query tiles would be
// almost empty, and it would read each kv head's cache once per query head.
//
// B200 design:
//   * One CTA per (batch, kv head, split of the key range): all G = Hq/Hkv query heads x Nq tokens
//     of that kv head (R = G * Nq rows, padded to RP = 16, 32 or 64) are served by one pass over
//     the cache, so every cached byte is read once (GQA-aware).  The key range of a sequence is
//     split across CTAs (split-KV) so that small batches still put enough SMs on the cache; the
//     splits are merged by their log-sum-exp in a second small kernel.
//   * The score tile is computed transposed, S^T = K Q^T (tcgen05.mma, M = 128 keys, N = RP query
//     rows): TMEM lane = key.  Each softmax thread owns one key and RP/NWG query columns; the
//     column maxima over the 128 keys take one redux.sync per column and warp plus a 4-warp
//     exchange in shared memory.  P^T is written to shared memory (16-bit, 128-byte swizzle) and
//     O^T += V^T P^T is a second MMA whose A operand is the V tile read MN-major, so TMEM lane =
//     output channel.  The row sums l stay per thread (per key lane) and are reduced once at the
//     end.
//   * K and V tiles (128 keys x 128 channels) stream through TMA rings with evict-first hints; the
//     next tile's S^T is computed while the softmax works on the current one (two S^T buffers).
//   * Cache entries past len_b are never used: their scores are masked and, in the last tile of a
//     sequence, their V rows are zeroed in shared memory before the P V product, so whatever the
//     cache holds there (NaN included) cannot reach the output.
//   * Lazy rescaling as in the prefill kernel (the running max moves only when a column's max
//     grows by more than 2^8), bounded waits everywhere, and a group-wide AND at every named
//     barrier so that a timeout makes all threads of a warpgroup leave together.
#pragma once
#include <climits>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ptx.cuh"

namespace tattn {

struct DecParams {
  int B, Hq, Hkv, Nq, Nk;
  int R;                 // (Hq / Hkv) * Nq query rows per kv head
  int causal;
  float scale_log2;      // scale * log2(e)
  const int* kv_lens;    // [B] cached keys per sequence (clamped to [0, Nk]); null: all Nk
  void* o;               // [B, Hq, Nq, 128] 16-bit
  float* lse;            // [B, Hq, Nq] or null
  // A unit split over several CTAs: each piece's partial result goes to slot u + i (CTA i), so
  // U + P - 1 slots cover every partition, and the CTA that finishes the unit's last piece
  // merges them (it learns that it is last from the unit's arrival counter, which it then resets
  // to zero, so a completed call leaves every counter at zero).
  float* part_o;         // [slots, R, 128] fp32, normalised per piece
  float* part_lse;       // [slots, R]
  unsigned int* unit_arrived;  // [U]
};

template <int RP>
struct DecCfg {
  static constexpr int D = 128;
  // Query columns per softmax thread: two warpgroups share every tile (each takes half of the
  // columns), so every SM sub-partition runs two softmax warps.
#ifndef TATTN_DEC_WG
#define TATTN_DEC_WG 2
#endif
  static constexpr int NWG_WANT = TATTN_DEC_WG < RP / 8 ? TATTN_DEC_WG : RP / 8;  // at least 8 columns
  static constexpr int NWG = RP / 32 > NWG_WANT ? RP / 32 : NWG_WANT;          // at most 32 columns
  static constexpr int CW = RP / NWG;
  static constexpr int kSoftmaxWarps = 4 * NWG;
  static constexpr int kTmaWarp = kSoftmaxWarps, kMmaWarp = kSoftmaxWarps + 1;
  static constexpr int kThreads = (kSoftmaxWarps + 2) * 32;
  static constexpr int PANEL = 128 * 128;        // 128 keys x 64 channels x 2 B (one TMA box)
  static constexpr int KV_TILE = 2 * PANEL;
  static constexpr int Q_PANEL = RP * 128, Q_TILE = 2 * Q_PANEL;  // two Q buffers (pieces alternate)
  static constexpr int P_PANEL = RP * 128, P_TILE = 2 * P_PANEL;  // RP rows x 64 keys x 2 B per panel
  static constexpr int KS = RP <= 32 ? 3 : 2;
  static constexpr int VS = RP <= 16 ? 3 : 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_P = OFF_Q + 2 * Q_TILE;
  static constexpr int OFF_K = OFF_P + 2 * P_TILE;
  static constexpr int OFF_V = OFF_K + KS * KV_TILE;
  static constexpr int OFF_RED = OFF_V + VS * KV_TILE;    // float [2][4][RP]: per-warp column maxima
  static constexpr int OFF_LRED = OFF_RED + 2 * RP * 16;  // float [RP][4] per-warp row sums, + 1 flag
  static constexpr int OFF_M = OFF_LRED + RP * 16 + 16;   // float [2][RP]: running column maxima
  static constexpr int OFF_SCHED = OFF_M + 2 * RP * 4;    // long long [8]: this CTA's tile range
  static constexpr int OFF_BAR = OFF_SCHED + 64;
  // q_full[2], q_empty[2], k_full[KS], k_empty[KS], v_full[VS], v_empty[VS], s_full[2], s_free[2],
  // p_full[2], o_done[2], o_final[2], o_free[2], drain
  static constexpr int NBAR = 4 + 2 * KS + 2 * VS + 12 + 1;
  static constexpr int SMEM_USED = OFF_BAR + NBAR * 8 + 16;
  static constexpr int SMEM_BYTES = SMEM_USED + 1024;
  static constexpr uint32_t TMEM_COLS = 4 * RP <= 64 ? 64u : (4 * RP <= 128 ? 128u : 256u);
  __host__ __device__ static constexpr uint32_t tm_s(int buf) { return (uint32_t)(buf * RP); }
  __host__ __device__ static constexpr uint32_t tm_o(int buf) { return (uint32_t)((2 + buf) * RP); }
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(RP % 16 == 0 && RP <= 64, "N of the M = 128 MMAs");
  static_assert(CW % 8 == 0, "the merge takes columns eight at a time");
};

enum : int { WD_LOAD = 0x60, WD_MMA = 0x70, WD_SOFTMAX = 0x80, WD_DRAIN = 0x90 };

// S^T(tmem, 128 keys x RP) = K_tile (128 x 128, K-major) * Q^T (Q: RP x 128, K-major); both staged
// by TMA with the 128-byte swizzle in two 64-channel panels.
template <int RP, bool FP16>
__device__ __forceinline__ void issue_kq(uint32_t s_tmem, uint32_t k_smem, uint32_t q_smem) {
  constexpr uint32_t idesc = instr_desc(1, FP16 ? 0 : 1, 0, 0, 128, RP);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {  // 16 channels (32 bytes) per MMA
    const uint32_t col = (uint32_t)(kk & 3) * 32;
    const uint64_t ad = smem_desc(k_smem + (kk >> 2) * DecCfg<RP>::PANEL + col, 16, 1024, kSwizzle128B);
    const uint64_t bd = smem_desc(q_smem + (kk >> 2) * DecCfg<RP>::Q_PANEL + col, 16, 1024, kSwizzle128B);
    mma_f16_ss(s_tmem, ad, bd, idesc, kk > 0 ? 1u : 0u);
  }
}

// O^T(tmem, 128 channels x RP) (+)= V^T (V_tile read MN-major: 64-channel panels 16 KB apart,
// 8-key groups 1024 B apart) * P^T (P: RP x 128 keys, K-major, two 64-key panels).
template <int RP, bool FP16>
__device__ __forceinline__ void issue_vp(uint32_t o_tmem, uint32_t v_smem, uint32_t p_smem, bool accumulate) {
  constexpr uint32_t idesc = instr_desc(1, FP16 ? 0 : 1, 1, 0, 128, RP);
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {  // 16 keys per MMA
    const uint64_t ad = smem_desc(v_smem + kk * 16 * 128, DecCfg<RP>::PANEL, 1024, kSwizzle128B);
    const uint64_t bd =
        smem_desc(p_smem + (kk >> 2) * DecCfg<RP>::P_PANEL + (uint32_t)(kk & 3) * 32, 16, 1024, kSwizzle128B);
    mma_f16_ss(o_tmem, ad, bd, idesc, (accumulate || kk > 0) ? 1u : 0u);
  }
}

template <bool FP16>
__device__ __forceinline__ uint16_t to16(float x) {
  if constexpr (FP16) return __half_as_ushort(__float2half_rn(x));
  else return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

template <int CW>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[CW]) {
  if constexpr (CW == 8) {
    tmem_ld8(taddr, r);
    tmem_ld_wait8(r);
  } else if constexpr (CW == 16) {
    tmem_ld16(taddr, r);
    tmem_ld_wait16(r);
  } else {
    tmem_ld32(taddr, r);
    tmem_ld_wait(r);
  }
}
template <int CW>
__device__ __forceinline__ void tmem_st_cols(uint32_t taddr, const uint32_t (&r)[CW]) {
  if constexpr (CW == 8) tmem_st8(taddr, r);
  else if constexpr (CW == 16) tmem_st16(taddr, r);
  else tmem_st32(taddr, r);
}

__device__ __forceinline__ int dec_len(const DecParams& p, int b) {
  const int len = p.kv_lens ? __ldg(&p.kv_lens[b]) : p.Nk;
  return min(max(len, 0), p.Nk);
}

// Walks this CTA's contiguous range [g, g_end) of the global key-tile sequence.  The sequence lists
// the units (batch b, kv head h) in order, each with ceil(len_b / 128) tiles; the part of the range
// that falls in one unit is a "piece".  Every role (producer, MMA issuer, softmax) runs its own
// copy of the cursor and so visits the same tiles in the same order.
struct DecCursor {
  int b, h, lt;          // current unit and local tile index in it
  int ps, pe;            // current piece: local tiles [ps, pe)
  int ntb, len;          // tiles and keys of batch b
  int k;                 // pieces started so far (selects the Q and O buffers)
  int gl;                // tiles visited so far (selects ring stages and S/P buffers)
  long long g, g_end;    // global index of tile lt; end of the CTA's range

  __device__ __forceinline__ void init(const DecParams& p, const long long* sched) {
    g = sched[0];
    g_end = sched[1];
    b = (int)sched[3];
    h = (int)sched[4];
    lt = (int)sched[5];
    k = 0;
    gl = 0;
    if (g < g_end) {
      len = dec_len(p, b);
      ntb = (len + 127) / 128;
      ps = lt;
      pe = (int)min((long long)ntb, (long long)lt + (g_end - g));
    }
  }
  __device__ __forceinline__ bool valid() const { return g < g_end; }
  __device__ __forceinline__ bool first() const { return lt == ps; }
  __device__ __forceinline__ bool last() const { return lt + 1 == pe; }
  __device__ __forceinline__ int unit(const DecParams& p) const { return b * p.Hkv + h; }
  __device__ __forceinline__ void next(const DecParams& p) {
    ++lt;
    ++g;
    ++gl;
    if (lt < pe || g >= g_end) return;
    ++k;  // next piece: the next unit that has tiles
    if (++h == p.Hkv) {
      h = 0;
      do {
        if (++b >= p.B) {  // (only if kv_lens changed during the call)
          g = g_end;
          return;
        }
        len = dec_len(p, b);
        ntb = (len + 127) / 128;
      } while (ntb == 0);
    }
    lt = 0;
    ps = 0;
    pe = (int)min((long long)ntb, g_end - g);
  }
};

// The CTA's share of the key tiles: with T tiles in all and P CTAs, CTA i takes
// [floor(i T / P), floor((i + 1) T / P)).  One warp scans kv_lens twice (total, then the unit that
// holds the first tile).  sched = {first, end, T, b, h, local tile}.
__device__ void dec_schedule(const DecParams& p, long long* sched, int lane) {
  const unsigned FULL = 0xffffffffu;
  long long total = 0;
  for (int base = 0; base < p.B; base += 32) {
    const int bb = base + lane;
    long long n = bb < p.B ? (long long)((dec_len(p, bb) + 127) / 128) * p.Hkv : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(FULL, n, o);
      if (lane >= o) n += y;
    }
    total += __shfl_sync(FULL, n, 31);
  }
  const long long P = gridDim.x, i = blockIdx.x;
  const long long g0 = total * i / P, g1 = total * (i + 1) / P;
  int fb = 0, fh = 0, flt = 0;
  if (g0 < g1) {
    long long run = 0;
    for (int base = 0; base < p.B; base += 32) {
      const int bb = base + lane;
      const int ntb = bb < p.B ? (dec_len(p, bb) + 127) / 128 : 0;
      const long long n = (long long)ntb * p.Hkv;
      long long incl = n;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const long long y = __shfl_up_sync(FULL, incl, o);
        if (lane >= o) incl += y;
      }
      const long long excl = run + incl - n;
      const unsigned hit = __ballot_sync(FULL, n > 0 && g0 >= excl && g0 < excl + n);
      if (hit) {
        const int src = __ffs(hit) - 1;
        const long long off = __shfl_sync(FULL, g0 - excl, src);
        const int nt_src = __shfl_sync(FULL, ntb, src);
        fb = base + src;
        fh = (int)(off / nt_src);
        flt = (int)(off % nt_src);
        break;
      }
      run += __shfl_sync(FULL, incl, 31);
    }
  }
  if (lane == 0) {
    sched[0] = g0;
    sched[1] = g1;
    sched[2] = total;
    sched[3] = fb;
    sched[4] = fh;
    sched[5] = flt;
  }
}

template <int RP, bool FP16>
__global__ void __launch_bounds__(DecCfg<RP>::kThreads, 1)
    attn_decode_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const DecParams p) {
  using C = DecCfg<RP>;
  constexpr int CW = C::CW;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* q_empty = q_full + 2;
  uint64_t* k_full = q_empty + 2;
  uint64_t* k_empty = k_full + C::KS;
  uint64_t* v_full = k_empty + C::KS;
  uint64_t* v_empty = v_full + C::VS;
  uint64_t* s_full = v_empty + C::VS;
  uint64_t* s_free = s_full + 2;
  uint64_t* p_full = s_free + 2;
  uint64_t* o_done = p_full + 2;
  uint64_t* o_final = o_done + 2;
  uint64_t* o_free = o_final + 2;
  uint64_t* drain = o_free + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sP = smem + C::OFF_P;
  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sV = smem + C::OFF_V;
  float* red = reinterpret_cast<float*>(smem + C::OFF_RED);
  float* lred = reinterpret_cast<float*>(smem + C::OFF_LRED);
  float* m_sh = reinterpret_cast<float*>(smem + C::OFF_M);
  long long* sched = reinterpret_cast<long long*>(smem + C::OFF_SCHED);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], C::kSoftmaxWarps);
      mbar_init(&p_full[i], C::kSoftmaxWarps);
      mbar_init(&o_done[i], 1);
      mbar_init(&o_final[i], 1);
      mbar_init(&o_free[i], C::kSoftmaxWarps);
    }
    for (int i = 0; i < C::KS; ++i) { mbar_init(&k_full[i], 1); mbar_init(&k_empty[i], 1); }
    for (int i = 0; i < C::VS; ++i) { mbar_init(&v_full[i], 1); mbar_init(&v_empty[i], 1); }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == C::kMmaWarp) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == C::kTmaWarp) {
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
    }
    dec_schedule(p, sched, lane);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const long long total_tiles = sched[2];

  if (warp == C::kTmaWarp) {
    // ================================ TMA producer ================================
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();  // every cached byte is read once
      DecCursor c;
      c.init(p, sched);
      int q_issued = 0, k_issued = 0, v_issued = 0;
      bool ok = true;
      while (c.valid()) {
        const int u = c.unit(p);
        if (c.first()) {  // a new piece: the unit's query rows
          const int qb = c.k & 1;
          if (!(ok = mbar_wait(&q_empty[qb], ((c.k >> 1) & 1) ^ 1, abort_flag, WD_LOAD + 0))) break;
          mbar_arrive_expect_tx(&q_full[qb], C::Q_TILE);
          for (int pn = 0; pn < 2; ++pn)
            tma_load_3d(sQ + qb * C::Q_TILE + pn * C::Q_PANEL, &tmQ, pn * 64, 0, u, &q_full[qb], pol);
          q_issued = c.k + 1;
        }
        const int ks = c.gl % C::KS, vs = c.gl % C::VS;
        const int key0 = c.lt * 128;
        if (!(ok = mbar_wait(&k_empty[ks], ((c.gl / C::KS) & 1) ^ 1, abort_flag, WD_LOAD + 1))) break;
        mbar_arrive_expect_tx(&k_full[ks], C::KV_TILE);
        for (int pn = 0; pn < 2; ++pn)
          tma_load_3d(sK + ks * C::KV_TILE + pn * C::PANEL, &tmK, pn * 64, key0, u, &k_full[ks], pol);
        k_issued = c.gl + 1;
        if (!(ok = mbar_wait(&v_empty[vs], ((c.gl / C::VS) & 1) ^ 1, abort_flag, WD_LOAD + 2))) break;
        mbar_arrive_expect_tx(&v_full[vs], C::KV_TILE);
        for (int pn = 0; pn < 2; ++pn)
          tma_load_3d(sV + vs * C::KV_TILE + pn * C::PANEL, &tmV, pn * 64, key0, u, &v_full[vs], pol);
        v_issued = c.gl + 1;
        c.next(p);
      }
      if (!ok) {
        // every issued copy must land before the CTA's shared memory is released
        for (int j = max(0, q_issued - 2); j < q_issued; ++j)
          mbar_wait(&q_full[j & 1], (j >> 1) & 1, nullptr, WD_DRAIN + 1, 200000000ull);
        for (int j = max(0, k_issued - C::KS); j < k_issued; ++j)
          mbar_wait(&k_full[j % C::KS], (j / C::KS) & 1, nullptr, WD_DRAIN + 2, 200000000ull);
        for (int j = max(0, v_issued - C::VS); j < v_issued; ++j)
          mbar_wait(&v_full[j % C::VS], (j / C::VS) & 1, nullptr, WD_DRAIN + 3, 200000000ull);
      }
    }
    __syncwarp();
  } else if (warp == C::kMmaWarp) {
    // ================================ MMA issuer ================================
    // Two in-order streams of tcgen05 work, issued by one thread as their inputs become ready:
    //   S^T(h) = K(h) Q^T   needs K(h), the piece's Q, and S^T buffer h % 2 read out (S^T(h - 2)),
    //   O^T += V^T P^T(g)   needs P^T(g), V(g) and, for a piece's first tile, its O buffer free.
    // Polling both with non-blocking tests keeps either stream from stalling behind the other
    // (S^T two tiles ahead often waits for its K tile while P^T is already there).
    if (lane == 0) {
      const uint32_t q_addr = smem_u32(sQ), p_addr = smem_u32(sP), k_addr = smem_u32(sK), v_addr = smem_u32(sV);
      DecCursor cs, cp;
      cs.init(p, sched);
      cp.init(p, sched);
      bool ok = true;
      unsigned long long t_idle = 0;
      uint32_t spins = 0;
      while (cp.valid()) {
        bool did = false;
        if (cs.valid()) {
          const int h = cs.gl, qb = cs.k & 1, ks = h % C::KS;
          if ((h < 2 || mbar_test(&s_free[h & 1], ((h - 2) >> 1) & 1)) &&
              (!cs.first() || mbar_test(&q_full[qb], (cs.k >> 1) & 1)) && mbar_test(&k_full[ks], (h / C::KS) & 1)) {
            tc_fence_after();
            issue_kq<RP, FP16>(tmem + C::tm_s(h & 1), k_addr + ks * C::KV_TILE, q_addr + qb * C::Q_TILE);
            mma_commit(&s_full[h & 1]);
            mma_commit(&k_empty[ks]);
            if (cs.last()) mma_commit(&q_empty[qb]);
            cs.next(p);
            did = true;
          }
        }
        {
          const int g = cp.gl, vs = g % C::VS, ob = cp.k & 1;
          if (cp.gl < cs.gl && mbar_test(&p_full[g & 1], (g >> 1) & 1) && mbar_test(&v_full[vs], (g / C::VS) & 1) &&
              (!cp.first() || mbar_test(&o_free[ob], ((cp.k >> 1) & 1) ^ 1))) {
            tc_fence_after();
            issue_vp<RP, FP16>(tmem + C::tm_o(ob), v_addr + vs * C::KV_TILE, p_addr + (g & 1) * C::P_TILE,
                               !cp.first());
            mma_commit(&v_empty[vs]);
            mma_commit(&o_done[g & 1]);  // one phase per two tiles
            if (cp.last()) mma_commit(&o_final[ob]);
            cp.next(p);
            did = true;
          }
        }
        // bounded: no progress for kWaitTimeoutNs (or another role's abort) ends the loop
        if (did) {
          spins = 0;
        } else if ((++spins & 63u) == 0u) {
          if (*abort_flag) { ok = false; break; }
          const unsigned long long now = globaltimer_ns();
          if (spins == 64u) t_idle = now;
          else if (now - t_idle > kWaitTimeoutNs) {
            report_timeout(abort_flag, WD_MMA + 7);
            ok = false;
            break;
          }
        }
      }
      if (!ok) {
        // every MMA issued so far must complete before TMEM is released
        mma_commit(drain);
        mbar_wait(drain, 0, nullptr, WD_DRAIN + 4, 200000000ull);
      }
    }
    __syncwarp();
  } else {
    // ================================ softmax ================================
    const int wg = warp >> 2, wq = warp & 3;
    const int t = wq * 32 + lane;    // TMEM lane: key t of the S^T tile, channel t of O^T
    const int c0 = wg * CW;          // first query column of this warpgroup
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    // one named barrier for all softmax warps: every decision taken on it is uniform across them
    constexpr int kBar = 1, kBarThreads = C::kSoftmaxWarps * 32;
    const int st = threadIdx.x;  // 0 .. kBarThreads - 1
    // rows of sequences without keys: O = 0, lse = -inf (no piece covers them)
    for (int bz = blockIdx.x; bz < p.B; bz += gridDim.x) {
      if (dec_len(p, bz) > 0) continue;
      const long long r0 = (long long)bz * p.Hq * p.Nq, nrow = (long long)p.Hq * p.Nq;
      for (long long e = st; e < nrow * 128; e += kBarThreads)
        reinterpret_cast<uint16_t*>(p.o)[r0 * 128 + e] = 0;
      if (p.lse != nullptr)
        for (long long e = st; e < nrow; e += kBarThreads) p.lse[r0 + e] = -INFINITY;
    }
    // P^T store address of element (row c, key t): two 64-key panels, 128-byte swizzle
    const uint32_t p_base = smem_u32(sP) + (uint32_t)(t >> 6) * C::P_PANEL + (uint32_t)(t & 7) * 2;
    const uint32_t p_chunk = (uint32_t)((t & 63) >> 3);
    float l_run[CW];
    bool ok = true;
    DecCursor cur;
    cur.init(p, sched);
    while (cur.valid()) {
      const int g = cur.gl, buf = g & 1;
      const bool first = cur.first();
      if (first) {
#pragma unroll
        for (int r = 0; r < CW; ++r) l_run[r] = 0.f;
      }
      const int len = cur.len;
      // Keys [0, lim(c)) are visible to query column c: lim = len, or under the causal mask
      // len - Nq + 1 + (c mod Nq).  Tiles that end at or before `edge` need no mask at all.
      // Padded columns (c >= R) are never masked: their Q rows are zeros, they only ever feed
      // their own columns of O^T and l, and nothing of them is written out.
      const int causal_base = len - p.Nq + 1;
      const int edge = p.causal ? min(len, causal_base) : len;
      bool okw = mbar_wait(&s_full[buf], (g >> 1) & 1, abort_flag, WD_SOFTMAX + 1);
      okw = __all_sync(0xffffffffu, okw);
      float s[CW];
      const int tile0 = cur.lt * 128;
      const int key = tile0 + t;
      if (okw) {
        tc_fence_after();
        uint32_t raw[CW];
        tmem_ld_cols<CW>(tmem + C::tm_s(buf) + (uint32_t)c0 + lane_off, raw);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_free[buf]);  // the MMA issuer may overwrite S^T(buf) now
#pragma unroll
        for (int r = 0; r < CW; ++r) s[r] = __uint_as_float(raw[r]);
        if (tile0 + 128 > edge) {  // (the same for the whole warpgroup)
#pragma unroll
          for (int r = 0; r < CW; ++r) {
            const int c = c0 + r;
            const int lim = p.causal ? causal_base + c % p.Nq : len;
            if (c < p.R && key >= lim) s[r] = -INFINITY;
          }
        }
      } else {
#pragma unroll
        for (int r = 0; r < CW; ++r) s[r] = -INFINITY;
      }
      {
        float wm[CW];
#pragma unroll
        for (int r = 0; r < CW; ++r) wm[r] = warp_max_f32(s[r]);
        if (lane == 0) {
          float4* dst = reinterpret_cast<float4*>(&red[(buf * 4 + wq) * RP + c0]);
#pragma unroll
          for (int q4 = 0; q4 < CW / 4; ++q4)
            dst[q4] = make_float4(wm[4 * q4], wm[4 * q4 + 1], wm[4 * q4 + 2], wm[4 * q4 + 3]);
        }
      }
      if (!(ok = named_bar_and(kBar, kBarThreads, okw && ok))) break;
      // Column maxima over the 128 keys and the lazy update of the running max m (kept in shared
      // memory, double-buffered by tile parity: every thread computes the same m, one thread
      // stores it).  Then P^T = exp2(s * scale_log2 - m), with masked keys giving exp2(-inf) = 0,
      // and the per-key partial row sums.
      // P^T(buf) was read by P V of tile g - 2: wait for phase (g - 2) / 2 of o_done[buf].  Every
      // tile waits for the next phase of one of the two barriers in turn, and P V of tile g needs
      // this tile's P^T, so the awaited phase is always the current or the last completed one.
      if (g >= 2) {
        bool okp = mbar_wait(&o_done[buf], ((g - 2) >> 1) & 1, abort_flag, WD_SOFTMAX + 5);
        ok = __all_sync(0xffffffffu, okp) && ok;
      }
      float alpha[CW];
      bool resc = false;
      const uint32_t pb = p_base + (uint32_t)buf * C::P_TILE;
      const float4* rd = reinterpret_cast<const float4*>(&red[buf * 4 * RP + c0]);
      const float4* mo = reinterpret_cast<const float4*>(&m_sh[(buf ^ 1) * RP + c0]);
      float4* mw = reinterpret_cast<float4*>(&m_sh[buf * RP + c0]);
#pragma unroll
      for (int q4 = 0; q4 < CW / 4; ++q4) {  // four columns at a time: vector loads of the maxima
        const float4 a = rd[q4], b4 = rd[RP / 4 + q4], c4 = rd[2 * (RP / 4) + q4], d4 = rd[3 * (RP / 4) + q4];
        const float4 m4 = first ? make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY) : mo[q4];
        const float wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b4.x, b4.y, b4.z, b4.w};
        const float wc[4] = {c4.x, c4.y, c4.z, c4.w}, wd[4] = {d4.x, d4.y, d4.z, d4.w};
        const float mold[4] = {m4.x, m4.y, m4.z, m4.w};
        float muse[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = 4 * q4 + i;
          const float mt = fmaxf(fmaxf(wa[i], wb[i]), fmaxf(wc[i], wd[i])) * p.scale_log2;
          const float mn = fmaxf(mold[i], mt);
          muse[i] = mold[i];
          alpha[r] = 1.f;
          if (mn > mold[i] + 8.f) {
            alpha[r] = ex2_approx(mold[i] - mn);
            muse[i] = mn;
            resc = true;
          }
        }
        if (wq == 0 && lane == 0) mw[q4] = make_float4(muse[0], muse[1], muse[2], muse[3]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = 4 * q4 + i, c = c0 + r;
          const float pv = ex2_approx(fmaf(s[r], p.scale_log2, muse[i] == -INFINITY ? 0.f : -muse[i]));
          l_run[r] = fmaf(l_run[r], alpha[r], pv);
          st_shared_u16(pb + (uint32_t)c * 128 + ((p_chunk ^ (uint32_t)(c & 7)) << 4), to16<FP16>(pv));
        }
      }
      // (resc and first are the same for every thread of the warpgroup)
      if (resc && !first) {
        // O^T must hold P V of the previous tile before it is rescaled: phase (g - 1) / 2 of
        // o_done[(g - 1) & 1] (the previous tile awaited its phase before, and P V of tile g + 1
        // waits for P^T(g + 1), so no later phase of that barrier can be done).
        bool oko = mbar_wait(&o_done[(g - 1) & 1], ((g - 1) >> 1) & 1, abort_flag, WD_SOFTMAX + 2);
        oko = __all_sync(0xffffffffu, oko);
        if (oko) {
          tc_fence_after();
          const uint32_t to = tmem + C::tm_o(cur.k & 1) + (uint32_t)c0 + lane_off;
          uint32_t o[CW];
          tmem_ld_cols<CW>(to, o);
#pragma unroll
          for (int r = 0; r < CW; ++r) o[r] = __float_as_uint(__uint_as_float(o[r]) * alpha[r]);
          tmem_st_cols<CW>(to, o);
          tmem_st_wait();
        }
        ok = oko;  // on failure the abort flag is raised: the next wait returns at once
      }
      // the sequence's last tile: zero the V rows of keys >= len (never valid cache entries)
      if (wg == 0 && tile0 + 128 > len) {
        const int vs = g % C::VS;
        const bool okv = mbar_wait(&v_full[vs], (g / C::VS) & 1, abort_flag, WD_SOFTMAX + 3);
        if (okv && key >= len) {
          const uint32_t vrow = smem_u32(sV) + (uint32_t)vs * C::KV_TILE + (uint32_t)t * 128;
#pragma unroll
          for (int pn = 0; pn < 2; ++pn)
#pragma unroll
            for (int q16 = 0; q16 < 8; ++q16) st_shared_zero16(vrow + pn * C::PANEL + q16 * 16);
        }
        ok = ok && okv;
      }
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[buf]);

      if (cur.last()) {
        // ---- end of a piece: reduce the row sums over the 128 keys, normalise, write the
        // piece's partial output and lse to slot (unit + CTA index) ----
        const int ob = cur.k & 1;
        bool oke = ok && mbar_wait(&o_final[ob], (cur.k >> 1) & 1, abort_flag, WD_SOFTMAX + 4);
#pragma unroll
        for (int r = 0; r < CW; ++r) {
          float v = l_run[r];
#pragma unroll
          for (int sh = 16; sh > 0; sh >>= 1) v += __shfl_xor_sync(0xffffffffu, v, sh);
          if (lane == 0) lred[(c0 + r) * 4 + wq] = v;
        }
        if (!(ok = named_bar_and(kBar, kBarThreads, oke))) break;
        tc_fence_after();
        uint32_t o[CW];
        tmem_ld_cols<CW>(tmem + C::tm_o(ob) + (uint32_t)c0 + lane_off, o);
        const int u = cur.unit(p);
        const float* m_last = m_sh + buf * RP;
        const long long row0 = (long long)u * p.R;  // output row of column 0 ((b, h, i) order)
        if (cur.ps == 0 && cur.pe == cur.ntb) {
          // the whole unit is this piece: final output
#pragma unroll
          for (int r = 0; r < CW; ++r) {
            const int c = c0 + r;
            if (c < p.R) {
              const float4 l4 = *reinterpret_cast<const float4*>(&lred[c * 4]);
              const float lsum = (l4.x + l4.y) + (l4.z + l4.w);
              reinterpret_cast<uint16_t*>(p.o)[(row0 + c) * 128 + t] =
                  to16<FP16>(lsum > 0.f ? __uint_as_float(o[r]) / lsum : 0.f);
              if (p.lse != nullptr && t == r)
                p.lse[row0 + c] = lsum > 0.f ? (m_last[c] + __log2f(lsum)) * 0.69314718055994531f : -INFINITY;
            }
          }
        } else {
          // a part of the unit: partial output (normalised) and lse to slot u + CTA index
          const long long slot = (long long)u + blockIdx.x;
#pragma unroll
          for (int r = 0; r < CW; ++r) {
            const int c = c0 + r;
            if (c < p.R) {
              const float4 l4 = *reinterpret_cast<const float4*>(&lred[c * 4]);
              const float lsum = (l4.x + l4.y) + (l4.z + l4.w);
              p.part_o[(slot * p.R + c) * 128 + t] = lsum > 0.f ? __uint_as_float(o[r]) / lsum : 0.f;
              if (t == r)
                p.part_lse[slot * p.R + c] =
                    lsum > 0.f ? (m_last[c] + __log2f(lsum)) * 0.69314718055994531f : -INFINITY;
            }
          }
          // The unit's tiles [g_u, g_u + n) lie in the CTAs i(g_u) .. i(g_u + n - 1), with
          // i(x) = ceil((x + 1) P / T) - 1; with fewer tiles than CTAs, empty shares hold nothing.
          const long long T = total_tiles, P = gridDim.x, gu = cur.g - cur.lt;
          const long long i_first = ((gu + 1) * P + T - 1) / T - 1;
          const long long i_last = ((gu + cur.ntb) * P + T - 1) / T - 1;
          // The barrier orders every thread's partial stores before thread 0's arrival, whose
          // release (cumulative over what the barrier ordered) publishes them GPU-wide; its
          // acquire makes the other pieces' partials visible to the CTA's merge below.
          named_bar_sync(kBar, kBarThreads);
          if (st == 0) {
            long long pieces = i_last - i_first + 1;
            if (T < P)
              for (long long i = i_first; i <= i_last; ++i) pieces -= (T * i / P == T * (i + 1) / P) ? 1 : 0;
            const unsigned int arrived = atom_add_acq_rel_gpu(&p.unit_arrived[u], 1u) + 1u;
            const bool last = arrived == (unsigned int)pieces;
            if (last) p.unit_arrived[u] = 0u;  // every piece has arrived: nothing else touches it this call
            lred[4 * RP] = last ? 1.f : 0.f;
          }
          named_bar_sync(kBar, kBarThreads);
          if (lred[4 * RP] != 0.f) {
            // merge: O = sum_i w_i O_i / sum_i w_i, w_i = exp(lse_i - max), lse = max + log(sum_i w_i),
            // running max over the pieces; 8 columns x 4 pieces of loads in flight at a time
            constexpr int MG = 8, KP = 4;
            for (int cg = 0; cg < CW; cg += MG) {
              float mx[MG], wsum[MG], acc[MG];
#pragma unroll
              for (int r = 0; r < MG; ++r) { mx[r] = -INFINITY; wsum[r] = 0.f; acc[r] = 0.f; }
              for (long long i = i_first; i <= i_last; i += KP) {
                float ls[KP][MG], ov[KP][MG];
#pragma unroll
                for (int kp = 0; kp < KP; ++kp) {
                  const long long ii = i + kp;
                  const bool have = ii <= i_last && !(T < P && T * ii / P == T * (ii + 1) / P);
                  const long long sl = (long long)u + ii;
#pragma unroll
                  for (int r = 0; r < MG; ++r) {
                    const int c = c0 + cg + r;
                    const bool use = have && c < p.R;
                    ls[kp][r] = use ? __ldcg(&p.part_lse[sl * p.R + c]) : -INFINITY;
                    ov[kp][r] = use ? __ldcg(&p.part_o[(sl * p.R + c) * 128 + t]) : 0.f;
                  }
                }
#pragma unroll
                for (int kp = 0; kp < KP; ++kp)
#pragma unroll
                  for (int r = 0; r < MG; ++r) {
                    const float l_i = ls[kp][r];
                    if (l_i == -INFINITY) continue;
                    if (l_i > mx[r]) {
                      const float sc = __expf(mx[r] - l_i);  // 0 for the first piece
                      acc[r] *= sc;
                      wsum[r] *= sc;
                      mx[r] = l_i;
                    }
                    const float w = __expf(l_i - mx[r]);
                    acc[r] = fmaf(w, ov[kp][r], acc[r]);
                    wsum[r] += w;
                  }
              }
#pragma unroll
              for (int r = 0; r < MG; ++r) {
                const int c = c0 + cg + r;
                if (c < p.R) {
                  reinterpret_cast<uint16_t*>(p.o)[(row0 + c) * 128 + t] =
                      to16<FP16>(wsum[r] > 0.f ? acc[r] / wsum[r] : 0.f);
                  if (p.lse != nullptr && t == 0)
                    p.lse[row0 + c] = wsum[r] > 0.f ? mx[r] + __logf(wsum[r]) : -INFINITY;
                }
              }
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&o_free[ob]);
      }
      cur.next(p);
    }
    tmem_st_wait();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace tattn
