// attn_fwd_kernels.cuh - the fused attention forward kernel for sm_100a (and the int32 score probe
// that shares its staging and MMA code).
//
// What it computes: O = softmax(scale * Q K^T [+ causal mask]) V and lse, per (batch, query head),
// with query head h reading kv head h / (Hq/Hkv) ("注意力即一切：从 MHA 到 GQA", sections 2.2, 2.3,
// 3.2, 5.1).  How: FlashAttention's tiling with an online softmax (same page, section 8.2; the
// "FlashAttention" glossary page, deep-dive section and FAQ): Q tiles stay on chip, K/V tiles stream
// through shared memory, a running row maximum m and row sum l rescale the partial output, and the
// N x N scores exist only as 128 x 128 tiles in tensor memory.  In INT8 mode the Q K^T tile is an
// INT8 x INT8 -> int32 product of the pre-pass outputs, dequantised by sq * sk (SageAttention
// article, section 技术方案), and P V stays in 16-bit floating point.  FP8 mode is the same with
// E4M3 codes and an fp32 product (tcgen05.mma kind::f8f6f4).
//
// B200 design (not the pages'; their kernels target Ampere/Ada/Hopper):
//   * CTA = 2 query tiles of 128 rows, 384 threads in four roles:
//       warps 0-3  softmax for query tile 0 (thread = one row; TMEM lanes 0..127)
//       warps 4-7  softmax for query tile 1
//       warp  8    TMA producer: Q tiles once, then K and V tiles through separate mbarrier rings
//       warp  9    MMA issuer (one thread): tcgen05.mma S = Q K^T into TMEM, O += P V from TMEM
//       warps 10-11 idle (they complete the producer warpgroup for the register split)
//     setmaxnreg moves registers from the producer warpgroup (56/thread) to the softmax
//     warpgroups (224/thread).
//   * TMEM (512 columns): S/P of tile t at column 128 t; O of tile t at column 256 + t D.
//     P (16-bit) is written over the first 64 columns of S and consumed as the A operand of P V
//     straight from TMEM, so P never touches shared memory.
//   * The two tiles ping-pong: while one softmax group works on its S, the tensor core runs the
//     other tile's P V and next Q K^T.
//   * Lazy rescaling: the running max used for exp2 moves only when a row's max grows by more than
//     2^8; otherwise the stale max keeps p <= 256 (exact: the same m is used for l and O).
//   * Every wait is bounded (ptx.cuh); a timeout raises a CTA abort flag, each role drains what it
//     has in flight and TMEM is always released.
#pragma once
#include <climits>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ptx.cuh"

namespace tattn {

// Query rows per work item: two 128-row tiles that ping-pong on the tensor cores (the default), or
// one tile (TATTN_QT1: a measurement variant showing what the second tile buys).
#ifndef TATTN_QT1
#define TATTN_QT1 0
#endif
constexpr int kItemRows = TATTN_QT1 ? 128 : 256;

struct FwdParams {
  int B, Hq, Hkv, N, causal;  // N: query rows
  int Nk;                 // keys (= N except under a row prefix mask)
  const int* row_lim;     // [N] or null: query row i sees keys j < row_lim[i] (clamped to [0, Nk])
  int n_mblocks;          // ceil(N / kItemRows)
  int sec_kv;             // kv heads per scheduling section (K/V of a section stay in L2)
  float scale_log2;       // scale * log2(e)
  void* o;                // [B, Hq, N, D] 16-bit
  float* lse;             // [B, Hq, N] or null
  const float* sq;        // 8-bit modes: [B, Hq, ceil(N/128)]
  const float* sk;        // 8-bit modes: [B, Hkv, ceil(N/128)]
  const float* bias;      // 8-bit modes: [B, Hq, N] (null allowed when lse is null)
};

// BYTE: Q and K staged as 1-byte codes (INT8 or FP8 modes), else 16-bit.
template <int D, bool BYTE>
struct FwdCfg {
  static constexpr int BM = 128, BN = 128, QT = 2;
  static constexpr int QK_ELEM = BYTE ? 1 : 2;                 // bytes per Q/K element
  static constexpr int QK_ROW = D * QK_ELEM;                   // bytes per Q/K row
  static constexpr int QK_SPAN = QK_ROW >= 128 ? 128 : 64;     // swizzle span (bytes)
  static constexpr uint32_t QK_SWZ = QK_SPAN == 128 ? kSwizzle128B : kSwizzle64B;
  static constexpr int QK_PANELS = QK_ROW / QK_SPAN;           // TMA boxes per tile
  static constexpr int QK_PANEL_BYTES = 128 * QK_SPAN;
  static constexpr int QK_BOX_X = QK_SPAN / QK_ELEM;           // elements per box row
  static constexpr int QK_STEPS = QK_ROW / 32;                 // 32 bytes of K per MMA
  static constexpr int Q_TILE = BM * QK_ROW;
  static constexpr int K_TILE = BN * QK_ROW;
  static constexpr int V_PANELS = D / 64;                      // 64 x 16-bit = 128 B per box row
  static constexpr int V_PANEL_BYTES = BN * 128;
  static constexpr int V_TILE = BN * D * 2;
  static constexpr int PV_STEPS = BN / 16;
  // Of every 16 score columns, how many take exp2_poly (FMA pipe) instead of MUFU ex2.  Measured
  // on the named workloads: it pays only where the exponentials outweigh the MMA work most
  // (d = 64: +3% in INT8 mode); at d = 128 every share tried was slower, so it is off there.
#ifndef TATTN_POLY_D128
#define TATTN_POLY_D128 0
#endif
#ifndef TATTN_POLY_D128_BYTE
#define TATTN_POLY_D128_BYTE TATTN_POLY_D128
#endif
#ifndef TATTN_POLY_D64
#define TATTN_POLY_D64 4
#endif
  static constexpr int POLY_PER_16 = D == 64 ? TATTN_POLY_D64 : (BYTE ? TATTN_POLY_D128_BYTE : TATTN_POLY_D128);
  // pipeline depth (K and V rings); defaults chosen by measurement on the named workloads
#ifndef TATTN_KS_128B
#define TATTN_KS_128B 2
#endif
#ifndef TATTN_VS_128B
#define TATTN_VS_128B 2
#endif
#ifndef TATTN_KS_128I
#define TATTN_KS_128I 4
#endif
#ifndef TATTN_VS_128I
#define TATTN_VS_128I 3
#endif
  // P in shared memory (compile-time alternative, 8-bit modes only, where the extra 64 KB fit): P of
  // query tile t lives in its own 128 x 128 16-bit buffer (K-major, 128-byte swizzle, two 64-key
  // panels) instead of over S in TMEM, so the next tile's Q K^T can overwrite S as soon as the
  // softmax has read it.  Measured 5-12% slower than P in TMEM on the named workloads: P V then
  // reads both operands from shared memory and the softmax writes P there, which doubles the
  // shared-memory traffic of a tile pair (about 256 KB instead of 128 KB, more cycles at 128 B/clk
  // than the pair's tensor work).  Off by default.
#ifndef TATTN_PSMEM
#define TATTN_PSMEM 0
#endif
  static constexpr bool PSMEM = BYTE && TATTN_PSMEM;
#ifndef TATTN_KS_PS128
#define TATTN_KS_PS128 3
#endif
#ifndef TATTN_VS_PS128
#define TATTN_VS_PS128 2
#endif
  static constexpr int KSTAGES = PSMEM ? (D == 128 ? TATTN_KS_PS128 : 4)
                                       : (D == 128 ? (BYTE ? TATTN_KS_128I : TATTN_KS_128B) : 4);
  static constexpr int VSTAGES = PSMEM ? (D == 128 ? TATTN_VS_PS128 : 4)
                                       : (D == 128 ? (BYTE ? TATTN_VS_128I : TATTN_VS_128B) : 4);
  static constexpr int P_PANEL_BYTES = 128 * 128;              // 128 rows x 64 keys x 2 B
  static constexpr int P_TILE = PSMEM ? 2 * P_PANEL_BYTES : 0;
  // O staging for the epilogue's TMA stores: one 32-row x 64-column 16-bit slot (4 KB, 128-byte
  // swizzle) per softmax warp; a warp stores its 32 rows panel by panel through its slot
  static constexpr int O_SLOT = 32 * 128;
  static constexpr int O_STAGE = PSMEM ? 0 : 8 * O_SLOT;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_P = OFF_Q + QT * Q_TILE;
  static constexpr int OFF_K = OFF_P + QT * P_TILE;
  static constexpr int OFF_V = OFF_K + KSTAGES * K_TILE;
  static constexpr int OFF_O = OFF_V + VSTAGES * V_TILE;
  static constexpr int OFF_BAR = OFF_O + O_STAGE;
  // barriers: q_full[2] k_full[KS] k_empty[KS] v_full[VS] v_empty[VS] s_full[2] p_full[2] o_done[2]
  // drain, then (P in shared memory) s_free[2] pv_done[2]
  static constexpr int NBAR = 2 + 2 * KSTAGES + 2 * VSTAGES + 6 + 1 + 4;
  static constexpr int SMEM_USED = OFF_BAR + NBAR * 8 + 32;  // + TMEM slot, abort flag, row-limit stats
  // +1024 for manual alignment of the dynamic shared memory base; at least 120 KB so that exactly
  // one CTA (which owns all 512 TMEM columns) is resident per SM.
  static constexpr int SMEM_BYTES = (SMEM_USED + 1024) > 120 * 1024 ? (SMEM_USED + 1024) : 120 * 1024;
  static constexpr uint32_t TMEM_COLS = 512;
  __host__ __device__ static constexpr uint32_t tm_s(int t) { return 128u * t; }
  __host__ __device__ static constexpr uint32_t tm_o(int t) { return 256u + (uint32_t)(D * t); }
  static_assert(SMEM_USED + 1024 <= 232448, "shared memory budget");
};

#ifndef TATTN_PFULL_PER_WARP
#define TATTN_PFULL_PER_WARP 1
#endif


// Warp roles.  Softmax warps come first, then one producer warpgroup (TMA warp, MMA warp, 2 idle).
//   SPLIT = false: 8 softmax warps, one thread per score row (32x32b TMEM accesses).
//   SPLIT = true : 16 softmax warps, four threads per score row (16x256b TMEM accesses): warps w
//                  and w+4 share a 32-lane TMEM quarter, 16 lanes each, and a row's max is
//                  reduced over its four threads with warp shuffles.  Each warp does half the
//                  exp2 work per tile, so a tile's softmax fits in the other tile's MMA time.
// setmaxnreg moves registers from the producer warpgroup to the softmax warpgroups; the split
// must fit the registers the CTA is launched with (65536 / threads, rounded down to 8).
template <bool SPLIT>
struct FwdRoles {
  static constexpr int kSoftmaxWarps = SPLIT ? 16 : 8;
  static constexpr int kThreads = (kSoftmaxWarps + 4) * 32;
  static constexpr int kLaunchRegs = (65536 / kThreads) / 8 * 8;
#ifndef TATTN_SPLIT_REGS_SOFTMAX
#define TATTN_SPLIT_REGS_SOFTMAX 104
#endif
#ifndef TATTN_SPLIT_REGS_PRODUCER
#define TATTN_SPLIT_REGS_PRODUCER 64
#endif
  static constexpr int kRegsSoftmax = SPLIT ? TATTN_SPLIT_REGS_SOFTMAX : 208;
  static constexpr int kRegsProducer = SPLIT ? TATTN_SPLIT_REGS_PRODUCER : 88;
  static constexpr int kTmaWarp = kSoftmaxWarps;
  static constexpr int kMmaWarp = kSoftmaxWarps + 1;
  static constexpr int kThreadsPerTile = kSoftmaxWarps * 16;  // softmax threads per query tile
  static_assert(128 * (kSoftmaxWarps / 4 * kRegsSoftmax + kRegsProducer) <= kThreads * kLaunchRegs,
                "register split exceeds the launch registers");
};

// Wait-site ids recorded with a timeout (role * 16 + barrier kind).
enum : int { W_LOAD = 0x10, W_MMA = 0x20, W_SOFTMAX = 0x30, W_DRAIN = 0x40, W_PROBE = 0x50 };

// Issue the QK_STEPS MMAs of S(tmem) = Q_tile * K_tile^T; both operands K-major, swizzled.
// Kind of the Q K^T product: 16-bit inputs (fp32 accumulate), INT8 codes (int32 accumulate) or
// FP8 E4M3 codes (fp32 accumulate).  The two 8-bit kinds share the 1-byte staging layout.
enum : int { QK_F16 = 0, QK_I8 = 1, QK_F8 = 2 };

template <int D, int QK, bool FP16>
__device__ __forceinline__ void issue_qk(uint32_t s_tmem, uint32_t q_smem, uint32_t k_smem) {
  constexpr bool INT8 = QK == QK_I8;
  using C = FwdCfg<D, QK != QK_F16>;
  constexpr uint32_t idesc = INT8             ? instr_desc(2, 1, 0, 0, 128, 128)
                             : QK == QK_F8 ? instr_desc(1, 0, 0, 0, 128, 128)  // E4M3 x E4M3 -> F32
                                           : instr_desc(1, FP16 ? 0 : 1, 0, 0, 128, 128);
  // one descriptor per operand; each K step adds its byte offset / 16 to the start-address field
  // (addresses stay below 256 KB, so the 14-bit field never carries)
  const uint64_t ad0 = smem_desc(q_smem, 16, 8 * C::QK_SPAN, C::QK_SWZ);
  const uint64_t bd0 = smem_desc(k_smem, 16, 8 * C::QK_SPAN, C::QK_SWZ);
#pragma unroll
  for (int kk = 0; kk < C::QK_STEPS; ++kk) {
    const uint32_t off = (uint32_t)((kk * 32) / C::QK_SPAN) * C::QK_PANEL_BYTES + (uint32_t)((kk * 32) % C::QK_SPAN);
    const uint64_t ad = ad0 + (off >> 4);
    const uint64_t bd = bd0 + (off >> 4);
    if constexpr (INT8)
      mma_i8_ss(s_tmem, ad, bd, idesc, kk > 0 ? 1u : 0u);
    else if constexpr (QK == QK_F8)
      mma_f8_ss(s_tmem, ad, bd, idesc, kk > 0 ? 1u : 0u);
    else
      mma_f16_ss(s_tmem, ad, bd, idesc, kk > 0 ? 1u : 0u);
  }
}

// Issue O(tmem) (+)= P(tmem, 16-bit, K-major) * V_tile(smem, MN-major, 128B swizzle).
template <int D, bool FP16>
__device__ __forceinline__ void issue_pv(uint32_t o_tmem, uint32_t p_tmem, uint32_t v_smem, bool accumulate) {
  constexpr uint32_t idesc = instr_desc(1, FP16 ? 0 : 1, 0, 1, 128, D);
  // 16 keys per step = 16 rows of 128 B; 64-column panels of V are 128 x 128 B apart (LBO),
  // groups of 8 key rows are 1024 B apart (SBO).  One descriptor; each step adds 2 KB / 16.
  const uint64_t bd0 = smem_desc(v_smem, 128 * 128, 1024, kSwizzle128B);
#pragma unroll
  for (int kk = 0; kk < 128 / 16; ++kk) {
    const uint64_t bd = bd0 + (uint64_t)(kk * 16 * 128 / 16);
    mma_f16_ts(o_tmem, p_tmem + kk * 8, bd, idesc, (accumulate || kk > 0) ? 1u : 0u);
  }
}

// 2^x on the FMA pipe (offloads the MUFU unit, which does one ex2 per score).  Range reduction
// 2^x = 2^n * 2^f with n = rint(x), f in [-1/2, 1/2] (Cody & Waite), then a degree-3 minimax
// polynomial for 2^f fitted with the Remez algorithm by tiled_attention_22_b200/exp2_fit.py
// (max relative error 7.5e-5 in float32 FMA arithmetic, below the 2^-9 rounding of 16-bit P).
// x is clamped at -125 so that adding n to the exponent field never leaves the normal range;
// softmax arguments here are <= 8 (lazy rescale), so there is no overflow side.
__device__ __forceinline__ float exp2_poly(float x) {
  x = fmaxf(x, -125.0f);
  const float t = x + 12582912.0f;  // 1.5 * 2^23: rint(x) lands in the low mantissa bits of t
  const float f = x - (t - 12582912.0f);
  float p = fmaf(5.517166853e-02f, f, 2.426111251e-01f);
  p = fmaf(p, f, 6.932609677e-01f);
  p = fmaf(p, f, 9.999280572e-01f);
  // the low 9 bits of t's pattern above the integer are zero, so (bits(t) << 23) == n << 23
  return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

// exp2_poly on a pair, with packed f32x2 arithmetic (10 issue slots per pair instead of 16).
__device__ __forceinline__ float2 exp2_poly2(float2 x);

__device__ __forceinline__ uint32_t pack2(float lo, float hi, bool fp16) {
  if (fp16) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  }
  __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&b);
}

__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
// Packed pair arithmetic (sm_100 f32x2): one instruction for two FP32 lanes.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;"
      : "=l"(d)
      : "l"(*reinterpret_cast<uint64_t*>(&a)), "l"(*reinterpret_cast<uint64_t*>(&b)),
        "l"(*reinterpret_cast<uint64_t*>(&c)));
  return *reinterpret_cast<float2*>(&d);
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;"
      : "=l"(d)
      : "l"(*reinterpret_cast<uint64_t*>(&a)), "l"(*reinterpret_cast<uint64_t*>(&b)));
  return *reinterpret_cast<float2*>(&d);
}

// One online-softmax step of one score row (this thread's row of the 128 x 128 tile in TMEM):
//   x = scores of the tile (fp32, or the int32 INT8 scores as 2^23*1.5 + acc, exact);
//   m_tile = max x * sc; the running max moves only when it grows by more than 8 (log2 units);
//   p = 2^(x*sc - m) rounded to 16 bits and stored over the first 64 columns of S (P V's A
//   operand); l accumulates the unrounded p; O is rescaled in TMEM when the max moved.
// MASKED: keys at tile columns >= lim are invisible (causal diagonal or past N): their x is
// -inf, so p = 2^-inf = 0 exactly (these tiles use MUFU ex2 for every column).
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  x.x = fmaxf(x.x, -125.0f);
  x.y = fmaxf(x.y, -125.0f);
  const float2 t = fadd2(x, make_float2(12582912.0f, 12582912.0f));
  const float2 n = fadd2(t, make_float2(-12582912.0f, -12582912.0f));
  const float2 f = ffma2(n, make_float2(-1.0f, -1.0f), x);  // x - n, exact
  float2 p = ffma2(make_float2(5.517166853e-02f, 5.517166853e-02f), f,
                   make_float2(2.426111251e-01f, 2.426111251e-01f));
  p = ffma2(p, f, make_float2(6.932609677e-01f, 6.932609677e-01f));
  p = ffma2(p, f, make_float2(9.999280572e-01f, 9.999280572e-01f));
  return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                     __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

// Row maximum of the tile's scores (raw: x, or 1.5*2^23 + acc for INT8 scores).
__device__ __forceinline__ float row_max128(const float (&x)[128]) {
  float mc[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    float m = x[32 * c];
#pragma unroll
    for (int k = 1; k < 31; k += 2) m = max3f(m, x[32 * c + k], x[32 * c + k + 1]);
    mc[c] = fmaxf(m, x[32 * c + 31]);
  }
  return max3f(mc[0], mc[1], fmaxf(mc[2], mc[3]));
}

// Row maximum of a tile of int32 scores (eight chains of two-input maxima).
__device__ __forceinline__ int row_max128_i32(const uint32_t (&r)[4][32]) {
  int mc[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    int m = max((int)r[c >> 1][(c & 1) * 16], (int)r[c >> 1][(c & 1) * 16 + 1]);
#pragma unroll
    for (int k = 2; k < 16; ++k) m = max(m, (int)r[c >> 1][(c & 1) * 16 + k]);
    mc[c] = m;
  }
  return max(max(max(mc[0], mc[1]), max(mc[2], mc[3])), max(max(mc[4], mc[5]), max(mc[6], mc[7])));
}

// INT8 scores, unmasked tiles, d = 128: the row maximum is taken on the int32 scores as loaded, and
// their conversion to float (one integer add each) is left to the exponential loop, where it
// overlaps the MUFU work instead of preceding the maximum.  Measured +2-4% on the 8192- and
// 131072-token workloads; at d = 64 (where the exponentials outweigh the MMA work twice over) it
// measured -2%, so d = 64 converts first.
#ifndef TATTN_I8_LATE
#define TATTN_I8_LATE 1
#endif

template <int D, int QK, bool FP16, bool MASKED>
__device__ __forceinline__ bool softmax_step(uint32_t tS, uint32_t tO, float sc, int lim, int j, float& m_run,
                                             float& l_run, uint64_t* o_done_t, volatile int* abort_flag) {
  constexpr bool INT8 = QK == QK_I8;  // int32 scores (the FP8 kind's are fp32 like the 16-bit one's)
  using C = FwdCfg<D, QK != QK_F16>;
  uint32_t r[4][32];
  float x[128];
  // INT8: exact int32 -> float for |acc| < 2^22 (here |acc| <= 128 * 127^2): x = 1.5*2^23 + acc
  auto to_x = [&](int c) {
#pragma unroll
    for (int i = 32 * c; i < 32 * c + 32; ++i) {
      const uint32_t bits = r[i >> 5][i & 31];
      x[i] = INT8 ? __uint_as_float(bits + 0x4B400000u) : __uint_as_float(bits);
      if (MASKED && i >= lim) x[i] = -INFINITY;
    }
  };
  constexpr bool LATE = INT8 && !MASKED && D == 128 && TATTN_I8_LATE;
  float m_tile;
#pragma unroll
  for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32 * c, r[c]);
#pragma unroll
  for (int c = 0; c < 4; ++c) tmem_ld_wait(r[c]);
  if (LATE) {
    m_tile = (float)row_max128_i32(r) * sc;  // |acc| < 2^22: exact
  } else {
#pragma unroll
    for (int c = 0; c < 4; ++c) to_x(c);
    const float mx = row_max128(x);
    m_tile = INT8 ? (mx - 12582912.0f) * sc : mx * sc;
  }
  // Each row decides for itself whether its running max moves (so its rounding never depends on
  // other rows); the TMEM rescale of O below is warp-uniform (.aligned), and rows that keep their
  // max multiply by exactly 1.
  const float m_new = fmaxf(m_run, m_tile);
  const bool need = m_new > m_run + 8.0f;
  const bool rescale = __any_sync(0xffffffffu, need);
  float alpha = 1.f;
  if (need) {
    alpha = ex2_approx(m_run - m_new);
    l_run *= alpha;
    m_run = m_new;
  }
  // exponent argument (x - off) * sc - m, off = 1.5*2^23 for INT8 (removed exactly by the add;
  // folding it into the constant would round off*sc + m per tile, shifting whole tiles)
  // (a row that has seen no key yet, possible only under a row prefix mask, keeps m = -inf: its
  // masked scores then give exp2(-inf - 0) = 0 rather than -inf + inf)
  const float m_use = m_run == -INFINITY ? 0.f : m_run;
  const float2 sc2 = make_float2(sc, sc), cst2 = make_float2(-m_use, -m_use);
  const float2 off2 = make_float2(-12582912.0f, -12582912.0f);
  float2 ls0 = make_float2(0.f, 0.f), ls1 = make_float2(0.f, 0.f);
  if (LATE) {
#pragma unroll
    for (int c = 0; c < 4; ++c) to_x(c);
  }
#pragma unroll
  for (int qtr = 0; qtr < 4; ++qtr) {
    uint32_t pk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int col = 32 * qtr + 2 * i;
      float2 xv = make_float2(x[col], x[col + 1]);
      if constexpr (INT8) xv = fadd2(xv, off2);
      const float2 a = ffma2(xv, sc2, cst2);
      float p0, p1;
      if (!MASKED && (col & 15) >= 16 - C::POLY_PER_16) {
        const float2 pp = exp2_poly2(a);
        p0 = pp.x;
        p1 = pp.y;
      } else {
        p0 = ex2_approx(a.x);
        p1 = ex2_approx(a.y);
      }
      if (i & 1)
        ls1 = fadd2(ls1, make_float2(p0, p1));
      else
        ls0 = fadd2(ls0, make_float2(p0, p1));
      pk[i] = pack2(p0, p1, FP16);
    }
    tmem_st16(tS + 16 * qtr, pk);
  }
  l_run += (ls0.x + ls0.y) + (ls1.x + ls1.y);
  if (rescale && j > 0) {
    // O holds the P V sums of key tiles 0..j-1.  The s_full commit that woke this thread was made
    // after S(j), i.e. after P V(j-1) was issued by the same thread, and a commit tracks every
    // earlier tcgen05 operation of its thread: P V(j-1) has completed.  P V(j) is issued only
    // after this thread arrives on p_full.
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t o[32];
      tmem_ld32(tO + 32 * c, o);
      tmem_ld_wait(o);
#pragma unroll
      for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
      tmem_st32(tO + 32 * c, o);
    }
  }
  return true;
}

// Split-row variant of softmax_step: this thread holds rows A (lane base + t/4) and B (+8), and
// of each row the columns 8k + 2(t%4) + {0,1}, k = 0..15 (a 16x256b TMEM load).  Row maxima are
// reduced over the 4 threads of a row with two xor-shuffles; each thread keeps a partial row sum
// (summed over the 4 threads in the epilogue).  P goes back with a 16x128b store, which puts the
// packed pair of columns (8k + 2(t%4), +1) at packed column 4k + t%4 of the same rows.
template <int D, int QK, bool FP16, bool MASKED>
__device__ __forceinline__ bool softmax_step_split(uint32_t tS, uint32_t tO, float sc, int limA, int limB, int j,
                                                   float (&m_run)[2], float (&l_run)[2], uint64_t* o_done_t,
                                                   volatile int* abort_flag) {
  constexpr bool INT8 = QK == QK_I8;
  const int q4 = threadIdx.x & 3;
  uint32_t r[64];
  tmem_ld_16x256_x16(tS, r);
  tmem_ld_wait64(r);
  float x[64];
#pragma unroll
  for (int i = 0; i < 64; ++i) {
    x[i] = INT8 ? __uint_as_float(r[i] + 0x4B400000u) : __uint_as_float(r[i]);
    if (MASKED) {
      const int col = 8 * (i >> 2) + 2 * q4 + (i & 1);
      if (col >= ((i & 2) ? limB : limA)) x[i] = -INFINITY;
    }
  }
  // repetitions 0..15: rep 0 starts the chains, reps (1,2) ... (13,14) in pairs, rep 15 alone
  float mA0 = x[0], mA1 = x[1], mB0 = x[2], mB1 = x[3];
#pragma unroll
  for (int k = 1; k + 1 < 16; k += 2) {
    mA0 = max3f(mA0, x[4 * k], x[4 * k + 4]);
    mA1 = max3f(mA1, x[4 * k + 1], x[4 * k + 5]);
    mB0 = max3f(mB0, x[4 * k + 2], x[4 * k + 6]);
    mB1 = max3f(mB1, x[4 * k + 3], x[4 * k + 7]);
  }
  float mx[2] = {max3f(mA0, mA1, x[60]), max3f(mB0, mB1, x[62])};
  mx[0] = fmaxf(mx[0], x[61]);
  mx[1] = fmaxf(mx[1], x[63]);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 1));
    mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xffffffffu, mx[h], 2));
  }
  float alpha[2] = {1.f, 1.f};
  bool need_any = false;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const float m_tile = INT8 ? (mx[h] - 12582912.0f) * sc : mx[h] * sc;
    const float m_new = fmaxf(m_run[h], m_tile);
    if (m_new > m_run[h] + 8.0f) {  // same decision in all 4 threads of the row
      alpha[h] = ex2_approx(m_run[h] - m_new);
      l_run[h] *= alpha[h];
      m_run[h] = m_new;
      need_any = true;
    }
  }
  const bool rescale = __any_sync(0xffffffffu, need_any);
  const float2 sc2 = make_float2(sc, sc);
  const float2 cA = make_float2(-m_run[0], -m_run[0]), cB = make_float2(-m_run[1], -m_run[1]);
  const float2 off2 = make_float2(-12582912.0f, -12582912.0f);
  float2 lsA = make_float2(0.f, 0.f), lsB = make_float2(0.f, 0.f);
  uint32_t pk[32];
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    float2 xa = make_float2(x[4 * k], x[4 * k + 1]);
    float2 xb = make_float2(x[4 * k + 2], x[4 * k + 3]);
    if constexpr (INT8) {
      xa = fadd2(xa, off2);
      xb = fadd2(xb, off2);
    }
    const float2 a = ffma2(xa, sc2, cA);
    const float2 b = ffma2(xb, sc2, cB);
    float pa0, pa1, pb0, pb1;
    if (!MASKED && (k & 7) >= 8 - FwdCfg<D, QK != QK_F16>::POLY_PER_16 / 2) {
      pa0 = exp2_poly(a.x);
      pa1 = exp2_poly(a.y);
      pb0 = exp2_poly(b.x);
      pb1 = exp2_poly(b.y);
    } else {
      pa0 = ex2_approx(a.x);
      pa1 = ex2_approx(a.y);
      pb0 = ex2_approx(b.x);
      pb1 = ex2_approx(b.y);
    }
    lsA = fadd2(lsA, make_float2(pa0, pa1));
    lsB = fadd2(lsB, make_float2(pb0, pb1));
    pk[2 * k] = pack2(pa0, pa1, FP16);
    pk[2 * k + 1] = pack2(pb0, pb1, FP16);
  }
  tmem_st_16x128_x16(tS, pk);
  l_run[0] += lsA.x + lsA.y;
  l_run[1] += lsB.x + lsB.y;
  if (rescale && j > 0) {
    // O holds the P V sums of key tiles 0..j-1.  The s_full commit that woke this thread was made
    // after S(j), i.e. after P V(j-1) was issued by the same thread, and a commit tracks every
    // earlier tcgen05 operation of its thread: P V(j-1) has completed.  P V(j) is issued only
    // after this thread arrives on p_full.
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      uint32_t o[32];
      tmem_ld_16x256_x8(tO + 64 * c, o);
      tmem_ld_wait(o);
#pragma unroll
      for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha[(i >> 1) & 1]);
      tmem_st_16x256_x8(tO + 64 * c, o);
    }
  }
  return true;
}

// Issue O(tmem) (+)= P(smem, 16-bit, K-major, 128-byte swizzle, two 64-key panels) * V_tile(smem,
// MN-major, 128-byte swizzle).
template <int D, bool FP16>
__device__ __forceinline__ void issue_pv_ss(uint32_t o_tmem, uint32_t p_smem, uint32_t v_smem, bool accumulate) {
  constexpr uint32_t idesc = instr_desc(1, FP16 ? 0 : 1, 0, 1, 128, D);
#pragma unroll
  for (int kk = 0; kk < 128 / 16; ++kk) {
    const uint64_t ad = smem_desc(p_smem + (kk >> 2) * (128 * 128) + (uint32_t)(kk & 3) * 32, 16, 1024, kSwizzle128B);
    const uint64_t bd = smem_desc(v_smem + kk * 16 * 128, 128 * 128, 1024, kSwizzle128B);
    mma_f16_ss(o_tmem, ad, bd, idesc, (accumulate || kk > 0) ? 1u : 0u);
  }
}

// softmax_step with P written to shared memory (see FwdCfg::PSMEM).  After S is in registers the
// warp arrives on s_free (the MMA issuer may overwrite S with the next tile's scores); before
// writing P it waits for P V of the previous tile (phase j - 1 of pv_done: every tile waits for
// the phase just before its own, so the awaited phase is never ambiguous), which also makes the
// O rescale safe.  p_row: shared address of this thread's row in panel 0 of the P buffer.
template <int D, int QK, bool FP16, bool MASKED>
__device__ __forceinline__ bool softmax_step_ps(uint32_t tS, uint32_t tO, float sc, int lim, int j, float& m_run,
                                                float& l_run, uint64_t* s_free_t, uint64_t* pv_done_t,
                                                uint32_t p_row, uint32_t p_xor, volatile int* abort_flag) {
  constexpr bool INT8 = QK == QK_I8;  // int32 scores
  const int lane = threadIdx.x & 31;
  uint32_t r[4][32];
#pragma unroll
  for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32 * c, r[c]);
#pragma unroll
  for (int c = 0; c < 4; ++c) tmem_ld_wait(r[c]);
  tc_fence_before();
  __syncwarp();
  if (lane == 0) mbar_arrive(s_free_t);
  float x[128];
#pragma unroll
  for (int i = 0; i < 128; ++i) {
    const uint32_t bits = r[i >> 5][i & 31];
    x[i] = INT8 ? __uint_as_float(bits + 0x4B400000u) : __uint_as_float(bits);
    if (MASKED && i >= lim) x[i] = -INFINITY;
  }
  float mc[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    float m = x[32 * c];
#pragma unroll
    for (int k = 1; k < 31; k += 2) m = max3f(m, x[32 * c + k], x[32 * c + k + 1]);
    mc[c] = fmaxf(m, x[32 * c + 31]);
  }
  const float mx = max3f(mc[0], mc[1], fmaxf(mc[2], mc[3]));
  const float m_tile = INT8 ? (mx - 12582912.0f) * sc : mx * sc;
  const float m_new = fmaxf(m_run, m_tile);
  const bool need = m_new > m_run + 8.0f;
  const bool rescale = __any_sync(0xffffffffu, need);
  float alpha = 1.f;
  if (need) {
    alpha = ex2_approx(m_run - m_new);
    l_run *= alpha;
    m_run = m_new;
  }
  const float m_use = m_run == -INFINITY ? 0.f : m_run;
  const float2 sc2 = make_float2(sc, sc), cst2 = make_float2(-m_use, -m_use);
  const float2 off2 = make_float2(-12582912.0f, -12582912.0f);
  float2 ls0 = make_float2(0.f, 0.f), ls1 = make_float2(0.f, 0.f);
  uint32_t pk[64];
#pragma unroll
  for (int i = 0; i < 64; ++i) {
    const int col = 2 * i;
    float2 xv = make_float2(x[col], x[col + 1]);
    if constexpr (INT8) xv = fadd2(xv, off2);
    const float2 a = ffma2(xv, sc2, cst2);
    const float p0 = ex2_approx(a.x), p1 = ex2_approx(a.y);
    if (i & 1)
      ls1 = fadd2(ls1, make_float2(p0, p1));
    else
      ls0 = fadd2(ls0, make_float2(p0, p1));
    pk[i] = pack2(p0, p1, FP16);
  }
  l_run += (ls0.x + ls0.y) + (ls1.x + ls1.y);
  if (j > 0) {
    bool ok = mbar_wait(pv_done_t, (j - 1) & 1, abort_flag, W_SOFTMAX + 5);
    if (!__all_sync(0xffffffffu, ok)) return false;
    tc_fence_after();
  }
  // 16-byte chunk c (8 keys) of the row goes to chunk c ^ (row % 8) of its panel row
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    const uint32_t a = p_row + (uint32_t)(c >> 3) * (128 * 128) + ((((uint32_t)c & 7u) ^ p_xor) << 4);
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(pk[4 * c]), "r"(pk[4 * c + 1]),
                 "r"(pk[4 * c + 2]), "r"(pk[4 * c + 3]));
  }
  if (rescale && j > 0) {
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t o[32];
      tmem_ld32(tO + 32 * c, o);
      tmem_ld_wait(o);
#pragma unroll
      for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
      tmem_st32(tO + 32 * c, o);
    }
  }
  return true;
}

template <int D, int QK, bool FP16, bool SPLIT>
__global__ void __launch_bounds__(FwdRoles<SPLIT>::kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                    const FwdParams p) {
  constexpr bool QUANT = QK != QK_F16;  // 8-bit codes with per-block scales sq, sk and the lse bias
  using C = FwdCfg<D, QUANT>;
  using R = FwdRoles<SPLIT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* k_full = q_full + 2;
  uint64_t* k_empty = k_full + C::KSTAGES;
  uint64_t* v_full = k_empty + C::KSTAGES;
  uint64_t* v_empty = v_full + C::VSTAGES;
  uint64_t* s_full = v_empty + C::VSTAGES;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_done = p_full + 2;
  uint64_t* drain = o_done + 2;
  uint64_t* s_free = drain + 1;    // P in shared memory only
  uint64_t* pv_done = s_free + 2;  // P in shared memory only
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(pv_done + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], TATTN_PFULL_PER_WARP ? R::kThreadsPerTile / 32 : R::kThreadsPerTile);
      mbar_init(&o_done[i], 1);
      mbar_init(&s_free[i], R::kThreadsPerTile / 32);
      mbar_init(&pv_done[i], 1);
    }
    for (int i = 0; i < C::KSTAGES; ++i) { mbar_init(&k_full[i], 1); mbar_init(&k_empty[i], 1); }
    for (int i = 0; i < C::VSTAGES; ++i) { mbar_init(&v_full[i], 1); mbar_init(&v_empty[i], 1); }
    mbar_init(drain, 1);
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

  // ---- work item: (m block of 256 query rows, batch, query head) ----
  // CTAs are ordered in sections of sec_kv consecutive (batch, kv head) pairs, sized on the host
  // so that a section's K and V fit comfortably in L2: all query heads and m blocks of a section
  // run close together and share those K/V tiles through L2.  Inside a section, m blocks go
  // heaviest first under causal masking (longest rows start first), query heads fastest.
  const int G = p.Hq / p.Hkv;
  const int n_bkv = p.B * p.Hkv;
  const int per_sec = p.sec_kv * G * p.n_mblocks;
  const int sec = (int)(blockIdx.x / (unsigned)per_sec);
  const int kv0 = sec * p.sec_kv;
  const int nkv_sec = min(p.sec_kv, n_bkv - kv0);
  const int rr = (int)blockIdx.x - sec * per_sec;
  const int mb_rank = rr / (nkv_sec * G);
  const int within = rr - mb_rank * (nkv_sec * G);
  const int kvz = kv0 + within / G;  // b * Hkv + kv head
  const int mb = (p.causal || p.row_lim) ? p.n_mblocks - 1 - mb_rank : mb_rank;
  const int b = kvz / p.Hkv;
  const int h = (kvz - b * p.Hkv) * G + within % G;
  const int bh = b * p.Hq + h;
  const int nkv = (p.Nk + 127) / 128;
  // Row prefix mask: the largest and smallest limit of each query tile's rows (rows < N), from
  // one warp, through shared memory: the largest sets the tile's key-tile count, the smallest
  // the first key tile that needs an element mask.
  int* lim_stats = reinterpret_cast<int*>(tmem_slot + 2);
  if (p.row_lim != nullptr) {
    if (warp == R::kTmaWarp) {
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        int mx = 0, mn = INT_MAX;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int row = mb * kItemRows + 128 * t + 32 * k + lane;
          if (row < p.N) {
            const int l = min(max(__ldg(&p.row_lim[row]), 0), p.Nk);
            mx = max(mx, l);
            mn = min(mn, l);
          }
        }
        mx = __reduce_max_sync(0xffffffffu, mx);
        mn = __reduce_min_sync(0xffffffffu, mn);
        if (lane == 0) {
          lim_stats[2 * t] = mx;
          lim_stats[2 * t + 1] = mn;
        }
      }
    }
    __syncthreads();
  }
  // key tiles each query tile visits (0 for a tile past N); n1 >= n0 unless tile 1 is empty
  auto key_tiles = [&](int t) {
    const int row0 = mb * kItemRows + 128 * t;
    if (row0 >= p.N || (TATTN_QT1 && t == 1)) return 0;
    if (p.row_lim != nullptr) return (lim_stats[2 * t] + 127) / 128;
    return p.causal ? min(nkv, row0 / 128 + 1) : nkv;
  };
  const int n0 = key_tiles(0), n1 = key_tiles(1);
  // (kept in registers: a runtime-indexed array would live in local memory)
  auto n_of = [&](int t) { return t ? n1 : n0; };
  const int nmax = max(n0, n1);

  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sV = smem + C::OFF_V;

  if (warp >= R::kSoftmaxWarps) {
    regs_decrease<R::kRegsProducer>();
  if (warp == R::kTmaWarp) {
    // ================================ TMA producer ================================
    if (lane == 0) {
      const uint64_t pol_stream = policy_evict_first();
      const uint64_t pol_keep = policy_evict_last();
      int k_issued = 0, v_issued = 0;
      bool ok = true;
      for (int t = 0; t < 2; ++t) {
        if (n_of(t) == 0) continue;
        mbar_arrive_expect_tx(&q_full[t], C::Q_TILE);
        for (int pn = 0; pn < C::QK_PANELS; ++pn)
          tma_load_3d(sQ + t * C::Q_TILE + pn * C::QK_PANEL_BYTES, &tmQ, pn * C::QK_BOX_X, mb * kItemRows + 128 * t, bh,
                      &q_full[t], pol_stream);
      }
      for (int j = 0; j < nmax && ok; ++j) {
        const int ks = j % C::KSTAGES, vs = j % C::VSTAGES;
        if (!(ok = mbar_wait(&k_empty[ks], ((j / C::KSTAGES) & 1) ^ 1, abort_flag, W_LOAD + 1))) break;
        mbar_arrive_expect_tx(&k_full[ks], C::K_TILE);
        for (int pn = 0; pn < C::QK_PANELS; ++pn)
          tma_load_3d(sK + ks * C::K_TILE + pn * C::QK_PANEL_BYTES, &tmK, pn * C::QK_BOX_X, j * 128, kvz,
                      &k_full[ks], pol_keep);
        k_issued = j + 1;
        if (!(ok = mbar_wait(&v_empty[vs], ((j / C::VSTAGES) & 1) ^ 1, abort_flag, W_LOAD + 2))) break;
        mbar_arrive_expect_tx(&v_full[vs], C::V_TILE);
        for (int pn = 0; pn < C::V_PANELS; ++pn)
          tma_load_3d(sV + vs * C::V_TILE + pn * C::V_PANEL_BYTES, &tmV, pn * 64, j * 128, kvz, &v_full[vs],
                      pol_keep);
        v_issued = j + 1;
      }
      if (!ok) {
        // Drain: every issued copy must land before the CTA's shared memory is released.
        for (int t = 0; t < 2; ++t)
          if (n_of(t)) mbar_wait(&q_full[t], 0, nullptr, W_DRAIN + 1, 200000000ull);
        for (int j = max(0, k_issued - C::KSTAGES); j < k_issued; ++j)
          mbar_wait(&k_full[j % C::KSTAGES], (j / C::KSTAGES) & 1, nullptr, W_DRAIN + 2, 200000000ull);
        for (int j = max(0, v_issued - C::VSTAGES); j < v_issued; ++j)
          mbar_wait(&v_full[j % C::VSTAGES], (j / C::VSTAGES) & 1, nullptr, W_DRAIN + 3, 200000000ull);
      }
    }
    __syncwarp();
  } else if (warp == R::kMmaWarp && C::PSMEM) {
    // ======================= MMA issuer, P in shared memory (event-driven) =======================
    // Four in-order streams: per query tile t, S_t(j) = Q_t K(j)^T (needs K(j) and S_t read out by
    // the softmax: s_free) and O_t += P_t(j) V(j) (needs P_t(j): p_full, and V(j)).  One thread
    // polls them with non-blocking tests and issues whatever is ready, so no stream waits behind
    // another.  A K or V stage is released after its last consumer (the later of the two tiles).
    if (lane == 0) {
      const uint32_t q_addr = smem_u32(sQ), k_addr = smem_u32(sK), v_addr = smem_u32(sV);
      const uint32_t p_addr = smem_u32(smem + C::OFF_P);
      int qj0 = 0, qj1 = 0, pj0 = 0, pj1 = 0;  // next Q K^T / P V index of each tile
      bool ok = true;
      unsigned long long t_idle = 0;
      uint32_t spins = 0;
      while (pj0 < n0 || pj1 < n1) {
        bool did = false;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
          const int nt = t ? n1 : n0, no = t ? n0 : n1;
          int& qj = t ? qj1 : qj0;
          int& pj = t ? pj1 : pj0;
          const int qo = t ? qj0 : qj1, po = t ? pj0 : pj1;
          if (pj < qj) {  // O_t += P_t(pj) V(pj)
            const int j = pj, vs = j % C::VSTAGES;
            if (mbar_test(&p_full[t], j & 1) && mbar_test(&v_full[vs], (j / C::VSTAGES) & 1)) {
              tc_fence_after();
              issue_pv_ss<D, FP16>(tmem + C::tm_o(t), p_addr + t * C::P_TILE, v_addr + vs * C::V_TILE, j > 0);
              mma_commit(&pv_done[t]);
              if (j + 1 == nt) mma_commit(&o_done[t]);  // the tile's last P V: O is final
              if (j >= no || po > j) mma_commit(&v_empty[vs]);  // the other tile is done with V(j)
              ++pj;
              did = true;
            }
          }
          if (qj < nt) {  // S_t(qj) = Q_t K(qj)^T
            const int j = qj, ks = j % C::KSTAGES;
            if ((j == 0 ? mbar_test(&q_full[t], 0) : mbar_test(&s_free[t], (j - 1) & 1)) &&
                mbar_test(&k_full[ks], (j / C::KSTAGES) & 1)) {
              tc_fence_after();
              issue_qk<D, QK, FP16>(tmem + C::tm_s(t), q_addr + t * C::Q_TILE, k_addr + ks * C::K_TILE);
              mma_commit(&s_full[t]);
              if (j >= no || qo > j) mma_commit(&k_empty[ks]);  // the other tile is done with K(j)
              ++qj;
              did = true;
            }
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
            report_timeout(abort_flag, W_MMA + 7);
            ok = false;
            break;
          }
        }
      }
      if (!ok) {
        // Drain: wait until every MMA issued so far has completed before TMEM is released.
        mma_commit(drain);
        mbar_wait(drain, 0, nullptr, W_DRAIN + 4, 200000000ull);
      }
    }
    __syncwarp();
  } else if (warp == R::kMmaWarp) {
    // ================================ MMA issuer ================================
    if (lane == 0) {
      const uint32_t q_addr = smem_u32(sQ), k_addr = smem_u32(sK), v_addr = smem_u32(sV);
      bool ok = true;
      auto users_first = [&](int j) { return j < n0 ? 0 : 1; };
      auto users_last = [&](int j) { return j < n1 ? 1 : 0; };
      // prologue: S_t(0) for both tiles
      if (nmax > 0) {
        ok = mbar_wait(&k_full[0], 0, abort_flag, W_MMA + 1);
        for (int t = 0; t < 2 && ok; ++t) {
          if (n_of(t) == 0) continue;
          if (!(ok = mbar_wait(&q_full[t], 0, abort_flag, W_MMA + 2))) break;
          tc_fence_after();
          issue_qk<D, QK, FP16>(tmem + C::tm_s(t), q_addr + t * C::Q_TILE, k_addr);
          mma_commit(&s_full[t]);
          if (users_last(0) == t) mma_commit(&k_empty[0]);
        }
      }
      for (int j = 0; j < nmax && ok; ++j) {
        const int vs = j % C::VSTAGES;
        const int ks1 = (j + 1) % C::KSTAGES;
        for (int t = 0; t < 2 && ok; ++t) {
          if (j >= n_of(t)) continue;
          // V(j) and K(j + 1) first (normally loaded long before), then P: once P is in, P V and
          // the next Q K^T go out with no further wait in between
          if (users_first(j) == t)
            if (!(ok = mbar_wait(&v_full[vs], (j / C::VSTAGES) & 1, abort_flag, W_MMA + 4))) break;
          if (j + 1 < n_of(t) && users_first(j + 1) == t)
            if (!(ok = mbar_wait(&k_full[ks1], ((j + 1) / C::KSTAGES) & 1, abort_flag, W_MMA + 5))) break;
          if (!(ok = mbar_wait(&p_full[t], j & 1, abort_flag, W_MMA + 3))) break;
          tc_fence_after();
          issue_pv<D, FP16>(tmem + C::tm_o(t), tmem + C::tm_s(t), v_addr + vs * C::V_TILE, j > 0);
          if (j + 1 == n_of(t)) mma_commit(&o_done[t]);  // the tile's last P V: O is final
          if (users_last(j) == t) mma_commit(&v_empty[vs]);
          if (j + 1 < n_of(t)) {
            issue_qk<D, QK, FP16>(tmem + C::tm_s(t), q_addr + t * C::Q_TILE, k_addr + ks1 * C::K_TILE);
            mma_commit(&s_full[t]);
            if (users_last(j + 1) == t) mma_commit(&k_empty[ks1]);
          }
        }
      }
      if (!ok) {
        // Drain: wait until every MMA issued so far has completed before TMEM is released.
        mma_commit(drain);
        mbar_wait(drain, 0, nullptr, W_DRAIN + 4, 200000000ull);
      }
    }
    __syncwarp();
  }  // remaining producer warps: nothing to do
  } else {
    regs_increase<R::kRegsSoftmax>();
    if constexpr (SPLIT) {
      // ============================ softmax, four threads per row ============================
      const int t = warp >> 3;                  // query tile
      const int wq = warp & 3;                  // TMEM lane quarter
      const int half = (warp >> 2) & 1;         // which 16 lanes of the quarter
      const int lane_base = wq * 32 + half * 16;
      const int nt = n_of(t);
      const int row0 = mb * kItemRows + 128 * t;
      const int rowA = row0 + lane_base + (lane >> 2), rowB = rowA + 8;
      const uint32_t tS = tmem + C::tm_s(t) + ((uint32_t)lane_base << 16);
      const uint32_t tO = tmem + C::tm_o(t) + ((uint32_t)lane_base << 16);
      const int nblk = (p.N + 127) / 128;
      const float sq_scale =
          (QUANT && nt > 0) ? p.sq[(size_t)bh * nblk + row0 / 128] * p.scale_log2 : p.scale_log2;
      float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
      bool ok = true;
      for (int j = 0; j < nt; ++j) {
        ok = mbar_wait(&s_full[t], j & 1, abort_flag, W_SOFTMAX + 1);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        float sc = QUANT ? sq_scale * __ldg(&p.sk[(size_t)kvz * nkv + j]) : sq_scale;
        if constexpr (QUANT) sc = fmaxf(sc, 1e-30f);
        const int col0 = j * 128;
        const bool diag = p.causal && (j == nt - 1);
        if (diag || (col0 + 128 > p.Nk)) {
          const int limA = (diag ? min(rowA + 1, p.Nk) : p.Nk) - col0;
          const int limB = (diag ? min(rowB + 1, p.Nk) : p.Nk) - col0;
          ok = softmax_step_split<D, QK, FP16, true>(tS, tO, sc, limA, limB, j, m_run, l_run, &o_done[t],
                                                       abort_flag);
        } else {
          ok = softmax_step_split<D, QK, FP16, false>(tS, tO, sc, 128, 128, j, m_run, l_run, &o_done[t],
                                                        abort_flag);
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
      if (ok && nt > 0) {
        ok = mbar_wait(&o_done[t], 0, abort_flag, W_SOFTMAX + 3);
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
          tc_fence_after();
          // full row sums: add the partials of the row's four threads
          float inv_l[2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 1);
            l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], 2);
            inv_l[h] = 1.0f / l_run[h];
          }
          const int q4 = lane & 3;
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            uint32_t o[32];
            tmem_ld_16x256_x8(tO + 64 * c, o);
            tmem_ld_wait(o);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const int col = 64 * c + 8 * k + 2 * q4;
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const int row = h ? rowB : rowA;
                const uint32_t v = pack2(__uint_as_float(o[4 * k + 2 * h]) * inv_l[h],
                                         __uint_as_float(o[4 * k + 2 * h + 1]) * inv_l[h], FP16);
                if (row < p.N)
                  *reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(p.o) +
                                               (((size_t)bh * p.N + row) * D + col) * 2) = v;
              }
            }
          }
          if (p.lse != nullptr && q4 == 0) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int row = h ? rowB : rowA;
              if (row < p.N) {
                float lse = (m_run[h] + __log2f(l_run[h])) * 0.69314718055994531f;
                if constexpr (QUANT) lse += p.bias[(size_t)bh * p.N + row];
                p.lse[(size_t)bh * p.N + row] = lse;
              }
            }
          }
        }
      }
      if (!ok) tmem_st_wait();
    } else {
      // ================================ softmax (one row per thread) ================================
      const int t = warp >> 2, wq = warp & 3;
      const int nt = n_of(t);
      const int row0 = mb * kItemRows + 128 * t;
      const int row = row0 + wq * 32 + lane;
      const uint32_t tS = tmem + C::tm_s(t) + ((uint32_t)(wq * 32) << 16);
      const uint32_t tO = tmem + C::tm_o(t) + ((uint32_t)(wq * 32) << 16);
      const int nblk = (p.N + 127) / 128;
      // (an empty tile, row0 >= N, reads nothing: its sq entry does not exist)
      const float sq_scale = (QUANT && nt > 0) ? p.sq[(size_t)bh * nblk + row0 / 128] * p.scale_log2 : p.scale_log2;
      float m_run = -INFINITY, l_run = 0.f;
      // row prefix mask: this row's limit, and the tile-wide smallest limit (rows < N)
      const int row_lim = (p.row_lim != nullptr && row < p.N) ? min(max(__ldg(&p.row_lim[row]), 0), p.Nk) : 0;
      const int tile_min_lim = p.row_lim != nullptr ? lim_stats[2 * t + 1] : INT_MAX;
      // (P in shared memory) this thread's row of the tile's P buffer, and its swizzle key
      const uint32_t p_row = smem_u32(smem + C::OFF_P) + (uint32_t)(t * C::P_TILE) + (uint32_t)(wq * 32 + lane) * 128u;
      const uint32_t p_xor = (uint32_t)(lane & 7);
      bool ok = true;
      // 8-bit modes: the key block's scale, loaded one tile ahead so that its latency is off the
      // tile's critical path
#ifndef TATTN_SK_PREFETCH
#define TATTN_SK_PREFETCH 1
#endif
      const float* skp = p.sk + (size_t)kvz * nkv;
      float sk_next = (QUANT && TATTN_SK_PREFETCH && nt > 0) ? __ldg(skp) : 0.f;
      // 8-bit modes: the row's lse bias, loaded now so that the epilogue does not wait for it
      const float lse_bias = (QUANT && p.lse != nullptr && nt > 0 && row < p.N) ? __ldg(&p.bias[(size_t)bh * p.N + row]) : 0.f;
      for (int j = 0; j < nt; ++j) {
        float sk_j = 0.f;
        if constexpr (QUANT) {
          if (TATTN_SK_PREFETCH) {
            sk_j = sk_next;
            if (j + 1 < nt) sk_next = __ldg(skp + j + 1);
          }
        }
        ok = mbar_wait(&s_full[t], j & 1, abort_flag, W_SOFTMAX + 1);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        if (QUANT && !TATTN_SK_PREFETCH) sk_j = __ldg(skp + j);
        float sc = QUANT ? sq_scale * sk_j : sq_scale;
        if constexpr (QUANT) sc = fmaxf(sc, 1e-30f);  // a zero block: keep -inf * sc = -inf for masks
        // causal diagonal tile (key > query), the ragged last key tile (key >= Nk) and, under a
        // row prefix mask, every tile that reaches past some row's limit are masked; keys
        // [0, lim) of the tile are visible
        const int col0 = j * 128;
        const bool diag = p.causal && (j == nt - 1);
        if constexpr (C::PSMEM) {
          if (diag || (col0 + 128 > p.Nk) || (col0 + 128 > tile_min_lim)) {
            const int lim = (p.row_lim != nullptr ? row_lim : (diag ? min(row + 1, p.Nk) : p.Nk)) - col0;
            ok = softmax_step_ps<D, QK, FP16, true>(tS, tO, sc, lim, j, m_run, l_run, &s_free[t], &pv_done[t], p_row,
                                                    p_xor, abort_flag);
          } else {
            ok = softmax_step_ps<D, QK, FP16, false>(tS, tO, sc, 128, j, m_run, l_run, &s_free[t], &pv_done[t],
                                                     p_row, p_xor, abort_flag);
          }
          if (!ok) break;
          fence_async_smem();  // P (generic stores) before the MMA's async-proxy reads
        } else {
          if (diag || (col0 + 128 > p.Nk) || (col0 + 128 > tile_min_lim)) {
            const int lim = (p.row_lim != nullptr ? row_lim : (diag ? min(row + 1, p.Nk) : p.Nk)) - col0;
            ok = softmax_step<D, QK, FP16, true>(tS, tO, sc, lim, j, m_run, l_run, &o_done[t], abort_flag);
          } else {
            ok = softmax_step<D, QK, FP16, false>(tS, tO, sc, 128, j, m_run, l_run, &o_done[t], abort_flag);
          }
          if (!ok) break;
        }
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
      if (ok && nt == 0 && p.row_lim != nullptr && row < p.N && !(TATTN_QT1 && t == 1)) {
        // every row of this tile sees no key: O = 0, lse = -inf
        uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint8_t*>(p.o) + ((size_t)bh * p.N + row) * (D * 2));
#pragma unroll
        for (int v = 0; v < D / 8; ++v) dst[v] = make_uint4(0u, 0u, 0u, 0u);
        if (p.lse != nullptr) p.lse[(size_t)bh * p.N + row] = -INFINITY;
      }
      if (ok && nt > 0) {
        ok = mbar_wait(&o_done[t], 0, abort_flag, W_SOFTMAX + 3);
        ok = __all_sync(0xffffffffu, ok);
        if (ok) {
          tc_fence_after();
          // (a row that saw no key, possible only under a row prefix mask, has l = 0: O = 0)
          const float inv_l = l_run > 0.f ? 1.0f / l_run : 0.f;
          if constexpr (C::O_STAGE > 0) {
            // O through this warp's shared-memory slot, one 64-column panel at a time, each
            // panel written to global memory by one TMA store of the warp's 32 rows (rows past
            // N are clipped by the tensor map).  Slot layout: row r at r * 128 bytes, 16-byte
            // chunk c at position c ^ (r & 7) (the 128-byte swizzle of the tensor map).
            uint8_t* slot = smem + C::OFF_O + warp * C::O_SLOT;
            const uint32_t swz = (uint32_t)(lane & 7);
            const int y0 = row0 + wq * 32;
#pragma unroll
            for (int pn = 0; pn < D / 64; ++pn) {
              if (pn > 0) {  // the previous panel's store has finished reading the slot
                if (lane == 0) bulk_wait_group_read0();
                __syncwarp();
              }
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
          } else {
            uint8_t* orow = reinterpret_cast<uint8_t*>(p.o) + ((size_t)bh * p.N + (size_t)row) * (D * 2);
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t o[32];
              tmem_ld32(tO + 32 * c, o);
              tmem_ld_wait(o);
              uint32_t pk[16];
#pragma unroll
              for (int i = 0; i < 16; ++i)
                pk[i] = pack2(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l, FP16);
              if (row < p.N) {
                uint4* dst = reinterpret_cast<uint4*>(orow + c * 64);
#pragma unroll
                for (int v = 0; v < 4; ++v)
                  dst[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
              }
            }
          }
          if (p.lse != nullptr && row < p.N) {
            float lse = l_run > 0.f ? (m_run + __log2f(l_run)) * 0.69314718055994531f : -INFINITY;
            if constexpr (QUANT) lse += lse_bias;
            p.lse[(size_t)bh * p.N + row] = lse;
          }
        }
      }
      if (!ok) {
        // make sure this thread's TMEM traffic is finished before teardown
        tmem_st_wait();
      }
      if constexpr (C::O_STAGE > 0) {
        // the slot must stay until the last store has read it
        if (lane == 0) bulk_wait_group_read0();
        __syncwarp();
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == R::kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------------------------------------
// Probe: int32 scores of selected (b, h, m_tile, n_tile) tiles through the same TMA staging
// (FwdCfg<D, true> layouts, same tensor maps) and the same issue_qk<D, true> MMA sequence.
// 160 threads: warps 0-3 read TMEM and write `out`, warp 4 loads and issues.
// ------------------------------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(160, 1)
    probe_qk_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK, int B, int Hq,
                    int Hkv, int N, const int32_t* tiles, int32_t* out) {
  using C = FwdCfg<D, true>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = smem + C::Q_TILE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::Q_TILE + C::K_TILE);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int tb = tiles[4 * blockIdx.x + 0], th = tiles[4 * blockIdx.x + 1];
  const int tm = tiles[4 * blockIdx.x + 2], tn = tiles[4 * blockIdx.x + 3];
  const int nblk = (N + 127) / 128;
  const bool valid = tb >= 0 && tb < B && th >= 0 && th < Hq && tm >= 0 && tm < nblk && tn >= 0 && tn < nblk;
  int32_t* dst = out + (size_t)blockIdx.x * 128 * 128;

  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 4) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    if (lane == 0 && valid) {
      const int kvz = tb * Hkv + th / (Hq / Hkv);
      mbar_arrive_expect_tx(&bars[0], C::Q_TILE + C::K_TILE);
      for (int pn = 0; pn < C::QK_PANELS; ++pn) {
        tma_load_3d(sQ + pn * C::QK_PANEL_BYTES, &tmQ, pn * C::QK_BOX_X, tm * 128, tb * Hq + th, &bars[0],
                    policy_evict_first());
        tma_load_3d(sK + pn * C::QK_PANEL_BYTES, &tmK, pn * C::QK_BOX_X, tn * 128, kvz, &bars[0],
                    policy_evict_first());
      }
      if (mbar_wait(&bars[0], 0, abort_flag, W_PROBE + 1)) {
        tc_fence_after();
        issue_qk<D, QK_I8, false>(tmem, smem_u32(sQ), smem_u32(sK));
      }
      mma_commit(&bars[1]);
    }
    __syncwarp();
  } else {
    const int row = warp * 32 + lane;
    bool ok = true;
    if (valid) {
      ok = mbar_wait(&bars[1], 0, abort_flag, W_PROBE + 2);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (valid && ok && !*abort_flag) {
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + 32 * c, r);
        tmem_ld_wait(r);
        uint4* d4 = reinterpret_cast<uint4*>(dst + (size_t)row * 128 + 32 * c);
#pragma unroll
        for (int v = 0; v < 8; ++v) d4[v] = make_uint4(r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]);
      }
    } else {
      uint4* d4 = reinterpret_cast<uint4*>(dst + (size_t)row * 128);
      for (int v = 0; v < 32; ++v) d4[v] = make_uint4(0, 0, 0, 0);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

}  // namespace tattn
