/*
 * tiled_attention.h - C ABI of the B200 (sm_100a) tiled attention forward pass.
 *
 * The operation (all entry points below compute parts of it):
 *
 *   O = softmax(scale * Q K^T [+ causal mask]) V,   lse_i = ln sum_j exp(s_ij)
 *
 *   "注意力即一切：从 MHA 到 GQA" (bojinhu.xyz), section 2.2 gives the four steps
 *   (scores Q K^T, softmax of the scaled scores, weighted sum of V), section
 *   2.3 the causal mask (future positions set to -inf before the softmax),
 *   section 3.2 the independent heads and section 5.1 the grouped K/V heads
 *   (GQA).  Section 8.2 of the same page and the "FlashAttention" glossary
 *   page (aiunderstanding.org; deep-dive section and FAQ) give the method:
 *   tiles of Q, K and V in on-chip memory with an online softmax (running row
 *   maximum and row sum, partial outputs rescaled), so the N x N score matrix
 *   never reaches HBM, and the result is the same as the plain definition.
 *
 *   ATTN_MODE_INT8_QK follows the SageAttention article "又快又准，即插即用！
 *   清华8比特量化Attention，两倍加速于FlashAttention2，各端到端任务均不掉点！",
 *   section 技术方案: K is smoothed by subtracting its per-channel mean over
 *   tokens, Q and K are quantised to INT8 with one scale per 128-token block,
 *   Q K^T runs on INT8 tensor cores with int32 accumulation and is dequantised,
 *   and P V stays in 16-bit floating point.
 *
 * Conventions shared by every entry point
 *   - Layout: dense row-major [B, H, N, d] (d fastest), H = Hq for Q and O,
 *     H = Hkv for K and V.  Query head h reads kv head h / (Hq / Hkv).
 *   - d must be 64 or 128.  N >= 1; N need not be a multiple of 128.
 *   - Every device pointer must be 16-byte aligned (TMA requirement).
 *   - All buffers belong to the caller.  The library allocates no memory.  Its
 *     own state, per GPU, is fixed-size device data built into the library:
 *     one device status word, 256 work-item counters of the persistent
 *     attention kernel (attn_fwd) and the 8 MiB K-mean array of
 *     attn_quant_smooth_k_noalloc.  The device addresses of the counters and
 *     of that array are looked up on first use on each device and cached, so
 *     the library must not be used across a cudaDeviceReset of that device.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream) and never synchronise, except attn_check_status and
 *     attn_fwd_host, which say so.
 *   - Inputs are never modified.
 *   - Return value: ATTN_OK (0) or a negative ATTN_ERR_* code.  Argument
 *     errors are detected on the host before anything is launched.
 *   - Device-side waits are bounded.  A wait that runs out sets the device
 *     status word; the kernel returns early and its outputs are undefined.
 *     attn_check_status() reports it as ATTN_ERR_TIMEOUT.
 */
#ifndef TILED_ATTENTION_H
#define TILED_ATTENTION_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum attn_status {
  ATTN_OK = 0,
  ATTN_ERR_ARG = -1,          /* null pointer, N < 1, Hq % Hkv != 0, bad scale/mode/dtype */
  ATTN_ERR_UNSUPPORTED = -2,  /* d not in {64, 128}, or sizes beyond 32-bit tensor indexing */
  ATTN_ERR_ALIGN = -3,        /* a device pointer is not 16-byte aligned */
  ATTN_ERR_WORKSPACE = -4,    /* workspace / scratch missing or smaller than required */
  ATTN_ERR_LAUNCH = -5,       /* a CUDA call or kernel launch failed (see attn_last_cuda_error) */
  ATTN_ERR_TIMEOUT = -6       /* a device-side wait ran out (reported by attn_check_status) */
};

enum attn_mode { ATTN_MODE_BF16_EXACT = 0, ATTN_MODE_INT8_QK = 1, ATTN_MODE_FP8_QK = 2 };
enum attn_dtype { ATTN_BF16 = 0, ATTN_FP16 = 1 };

/*
 * attn_fwd - the whole forward pass.
 *
 *   q [B,Hq,N,d], k [B,Hkv,N,d], v [B,Hkv,N,d]: device, dtype `dtype`.
 *   o [B,Hq,N,d]: device, written, dtype `dtype`.
 *   lse [B,Hq,N]: device float32, written; NULL skips it.  In INT8 mode lse
 *     includes the term scale*q_i.mean(K) that smoothing removes, so it is
 *     the log-sum-exp of the caller's scores in both modes.
 *   causal: 0 or 1 (key j is visible to query i when j <= i).
 *   scale: the softmax scale (finite, > 0), normally 1/sqrt(d).
 *   mode: ATTN_MODE_BF16_EXACT (16-bit Q K^T on tensor cores, fp32
 *     accumulation), ATTN_MODE_INT8_QK (runs the pre-pass of
 *     attn_quant_smooth_k into `workspace`, then INT8 Q K^T) or
 *     ATTN_MODE_FP8_QK (the pre-pass of attn_quant_smooth_k_fp8, then FP8
 *     E4M3 Q K^T with fp32 accumulation; same workspace size as INT8).
 *   workspace / ws_bytes: device memory of at least
 *     attn_workspace_bytes(B,Hq,Hkv,N,d,mode) bytes (0 for BF16_EXACT, where
 *     workspace may be NULL).  Its content on entry does not matter.
 *   Launches: BF16_EXACT with d = 128 runs on persistent CTAs (one per SM)
 *     that take 256-row work items from a counter inside the library, cleared
 *     by a 4-byte cudaMemsetAsync on the stream before the kernel.  There is
 *     one counter per stream, told apart by the stream's process-unique id
 *     (cudaStreamGetId), so cudaStreamPerThread used from several host
 *     threads, or a new stream that reuses a destroyed stream's handle value,
 *     gets its own counter; calls on one stream are ordered by the stream.
 *     A device has 256 counters; calls from further streams, and every call
 *     made while its stream is being captured into a CUDA graph (a captured
 *     counter address would be shared by every replay, on any stream), launch
 *     one CTA per work item instead, with the same results.  The first call on
 *     a device looks up the counters' address (with that device current):
 *     make it before any stream capture on the device.  The other modes and
 *     d = 64 launch one CTA per work item.
 */
int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
             int B, int Hq, int Hkv, int N, int d, int causal, float scale, int mode,
             int dtype, void* workspace, size_t ws_bytes, void* stream);

/* Bytes of workspace attn_fwd needs for these sizes and mode (0 for BF16_EXACT; the 8-bit modes
 * need the same). */
size_t attn_workspace_bytes(int B, int Hq, int Hkv, int N, int d, int mode);

/*
 * attn_quant_smooth_k - the INT8 pre-pass alone (SageAttention article,
 * section 技术方案, items on K smoothing and per-block INT8 quantisation).
 *
 *   kmean [B,Hkv,d] float32: per channel mean of K over all N tokens.  Sum
 *     order (reproducible bit for bit): within each 128-token block the tokens
 *     are added in ascending order into a float64 partial; the partials are
 *     added in ascending block order into a float64 total; the mean is
 *     (float)(total / N).
 *   k8 [B,Hkv,N,d] int8, sk [B,Hkv,ceil(N/128)] float32: ks = (float)k - kmean;
 *     per 128-token block (all d channels) amax = max|ks|, sk = amax/127,
 *     k8 = clamp(rint(ks * (127/amax)), -127, 127), ties to even; an all-zero
 *     block gives sk = 0 and k8 = 0.
 *   q8 [B,Hq,N,d] int8, sq [B,Hq,ceil(N/128)] float32: the same per-block
 *     quantisation applied to Q without smoothing.
 *   lse_bias [B,Hq,N] float32: scale * sum_c q[i,c] * kmean[g(h),c].
 *   scratch / scratch_bytes: device memory of at least
 *     attn_quant_scratch_bytes(B,Hkv,N,d) bytes (float64 block partials).
 *   q8, sq, k8, sk, kmean and lse_bias are device buffers written by the call.
 */
int attn_quant_smooth_k(const void* q, const void* k, int B, int Hq, int Hkv, int N, int d,
                        int dtype, float scale, int8_t* q8, float* sq, int8_t* k8, float* sk,
                        float* kmean, float* lse_bias, void* scratch, size_t scratch_bytes,
                        void* stream);

/* Bytes of scratch attn_quant_smooth_k needs: B*Hkv*ceil(N/128)*d*8 (+ alignment). */
size_t attn_quant_scratch_bytes(int B, int Hkv, int N, int d);

/*
 * attn_quant_smooth_k_fp8 - the pre-pass of ATTN_MODE_FP8_QK: the same K mean, smoothing and lse
 * bias as attn_quant_smooth_k, with FP8 E4M3 codes in place of INT8 ones.  The SageAttention
 * article (section 技术方案) weighs INT8 against FP8 for the 8-bit Q K^T; the FP8 variant keeps
 * its smoothing and per-block scales:
 *   per 128-token block (all d channels) amax = max|x|, scale = amax/448 (448 = largest finite
 *   E4M3), code = E4M3(fl32(x * (448/amax))), rounded to nearest with ties to even and
 *   saturated at +-448; an all-zero block has scale 0 and codes 0.
 *   q8 [B,Hq,N,d], k8 [B,Hkv,N,d]: E4M3 bit patterns (1 sign, 4 exponent bits with bias 7,
 *   3 mantissa bits, no infinities).  Other arguments as for attn_quant_smooth_k (same
 *   scratch size).
 */
int attn_quant_smooth_k_fp8(const void* q, const void* k, int B, int Hq, int Hkv, int N, int d,
                            int dtype, float scale, uint8_t* q8, float* sq, uint8_t* k8, float* sk,
                            float* kmean, float* lse_bias, void* scratch, size_t scratch_bytes,
                            void* stream);

/*
 * attn_fwd_fp8_quantized - the fused FP8 attention kernel alone, on the outputs of
 * attn_quant_smooth_k_fp8: S = E4M3 Q K^T with fp32 accumulation (tcgen05.mma kind::f8f6f4),
 * dequantised by sq * sk, online softmax, 16-bit P V.  Arguments as attn_fwd_int8_quantized.
 */
int attn_fwd_fp8_quantized(const uint8_t* q8, const float* sq, const uint8_t* k8,
                           const float* sk, const float* lse_bias, const void* v, void* o,
                           float* lse, int B, int Hq, int Hkv, int N, int d, int causal,
                           float scale, int dtype, void* stream);

/*
 * attn_quant_smooth_k_noalloc - the same pre-pass as attn_quant_smooth_k, for callers that cannot
 * allocate device memory: code that runs under another owner's memory pool that hands out no
 * extra device buffers, or a latency-bound loop that cannot afford cudaMalloc (which may
 * synchronise the whole device).  (The pages have no counterpart: this is an interface choice.)
 *
 *   Arguments and results are those of attn_quant_smooth_k without scratch / scratch_bytes: the
 *   caller still passes q, k and every output buffer.  The float64 K-mean partials go to an
 *   8 MiB array built into the library; each GPU that loads the library keeps its copy until the
 *   process exits.  Sizes are limited to B*Hkv*ceil(N/128)*d <= 1048576 (e.g. B=1, Hkv=8,
 *   N=131072, d=128); larger sizes return ATTN_ERR_WORKSPACE before launching (text in
 *   attn_last_cuda_error) and need attn_quant_smooth_k.
 *   The first call on each device looks up the array's device address (with that device
 *   current) and caches it; make that first call before any stream capture on that device, and
 *   do not use the library across a cudaDeviceReset of that device (the cached address would
 *   be stale).  The call itself allocates nothing.  All calls on a device share the one array, and it keeps
 *   the previous call's contents (every entry a call reads is written by the same call first):
 *   calls whose kernels overlap on the GPU (different streams, no ordering) race on it, so order
 *   them, for example by issuing them on one stream.
 */
int attn_quant_smooth_k_noalloc(const void* q, const void* k, int B, int Hq, int Hkv, int N, int d,
                                int dtype, float scale, int8_t* q8, float* sq, int8_t* k8,
                                float* sk, float* kmean, float* lse_bias, void* stream);

/*
 * attn_fwd_int8_quantized - the fused INT8 attention kernel alone, on the
 * outputs of attn_quant_smooth_k (q8, sq, k8, sk, lse_bias; all device).
 * v, o and lse as in attn_fwd.  lse_bias may be NULL only when lse is NULL.
 */
int attn_fwd_int8_quantized(const int8_t* q8, const float* sq, const int8_t* k8,
                            const float* sk, const float* lse_bias, const void* v, void* o,
                            float* lse, int B, int Hq, int Hkv, int N, int d, int causal,
                            float scale, int dtype, void* stream);

/*
 * attn_probe_qk_int32 - test hook: the exact int32 scores S = q8 k8^T of
 * selected 128x128 tiles, computed by the same TMA staging and INT8 tcgen05
 * MMA code the fused kernel uses, written to `out` instead of being
 * dequantised.
 *   tiles: device int32 array of 4*ntiles entries (b, h, m_tile, n_tile); the
 *     tile covers query rows [128*m_tile, +128) and keys [128*n_tile, +128)
 *     of query head h (kv head h / (Hq/Hkv)).  Each index is checked on the
 *     device; an out-of-range tile writes zeros.
 *   out: device int32 [ntiles, 128, 128]; rows/columns past N hold the
 *     scores of zero-filled rows (0).
 */
int attn_probe_qk_int32(const int8_t* q8, const int8_t* k8, int B, int Hq, int Hkv, int N,
                        int d, const int32_t* tiles, int ntiles, int32_t* out, void* stream);

/*
 * attn_fwd_host - attn_fwd with HOST buffers: copies q, k, v from host memory into the caller's
 * device buffers dq, dk, dv, runs the forward pass into do_ / dlse, and copies o (and lse when
 * both lse pointers are non-NULL) back to host memory; returns when the host outputs are ready.
 * The work is split into at most 10 pieces, each a run of query heads: piece c's inputs are
 * copied in on a helper stream while earlier pieces compute on `stream`, and outputs are copied
 * out on a second helper stream (two streams and per-piece events are created and destroyed by
 * the call; no device memory is allocated).  When N % 4 == 0 the first and last pieces are one
 * query head each (one (batch, kv head) unit when Hq == Hkv), so that little copying is left
 * outside the compute; the (batch, kv head) units between them form up to six pieces.  Otherwise
 * the pieces are up to 8 runs of whole units.  Outputs are bit-identical to attn_fwd's.  Host
 * buffers should be pinned for the copies to overlap.  One cudaMemcpyAsync per buffer per piece.
 * The 8-bit modes need workspace of at least attn_workspace_bytes(B,Hq,Hkv,N,d,mode) bytes (pieces
 * reuse it in turn).
 */
int attn_fwd_host(const void* q, const void* k, const void* v, void* o, float* lse,
                  void* dq, void* dk, void* dv, void* do_, float* dlse,
                  int B, int Hq, int Hkv, int N, int d, int causal, float scale, int mode,
                  int dtype, void* workspace, size_t ws_bytes, void* stream);

/*
 * attn_fwd_prefix_masked - attention in which query row i sees the keys j < row_kv_limit[i]
 * (a per-row visible prefix; the same limits for every batch and head), bf16/fp16 exact mode.
 * This is the mask of the APB article ("在长文本上比Flash Attention快10倍！清华等提出APB序列并行推理
 * 框架", sections on the anchor block, the passing block and the computation step, which uses a
 * special FlashAttention kernel with a changed mask): with keys laid out as
 * [anchor A | passing P | local L] and queries as [anchor A | local L], anchor row i has limit
 * i + 1 and local row i has limit A + P + i + 1.  Plain causal attention is limit i + 1.
 *   q [B, Hq, Nq, d]; k, v [B, Hkv, Nk, d]; o [B, Hq, Nq, d]; lse [B, Hq, Nq] or NULL.
 *   row_kv_limit: device int32 [Nq], 4-byte aligned; values are clamped to [0, Nk].  A row with
 *   limit 0 sees no key and gets O = 0, lse = -inf.  Key tiles past a query tile's largest
 *   limit are skipped.  d = 64 or 128.
 */
int attn_fwd_prefix_masked(const void* q, const void* k, const void* v, void* o, float* lse,
                           int B, int Hq, int Hkv, int Nq, int Nk, int d,
                           const int32_t* row_kv_limit, float scale, int dtype, void* stream);

/*
 * attn_decode - attention of Nq new query tokens per sequence against a KV cache (decoding, or
 * verifying a few drafted tokens).  "注意力即一切：从 MHA 到 GQA", section 3.4: with a KV cache the
 * keys and values of earlier tokens are stored, and each new token's query attends to all of
 * them; sections 2.2, 2.3 and 5.1 as above for the softmax, the mask and the head grouping.
 *
 *   q       [B, Hq, Nq, d]       the new tokens' queries (16-bit, dtype)
 *   k_cache [B, Hkv, Nk, d]      cached keys; sequence b uses its first kv_lens[b] positions
 *   v_cache [B, Hkv, Nk, d]      cached values, same layout
 *   kv_lens device int32 [B], or NULL (every sequence holds Nk keys).  Values are clamped to
 *           [0, Nk].  Cache entries at or past kv_lens[b] are never used, whatever they hold.
 *   o       [B, Hq, Nq, d]       output (dtype);  lse  [B, Hq, Nq] float (natural log) or NULL.
 *   causal  0: every new token sees all kv_lens[b] keys.  1: the new tokens are the LAST Nq of
 *           the kv_lens[b] positions, so token i sees keys 0 .. kv_lens[b] - Nq + i.  A row that
 *           sees no key (kv_lens[b] = 0, or kv_lens[b] < Nq under the mask) gets O = 0 and
 *           lse = -inf.
 *   d must be 128 and (Hq / Hkv) * Nq <= 64 (ATTN_ERR_UNSUPPORTED otherwise); 1 <= Nq <= Nk.
 *   num_ctas: persistent CTAs (0: one per SM of the current device).  All key tiles of all
 *           (batch, kv head) units form one sequence, and CTA i of P takes the contiguous share
 *           [floor(i T / P), floor((i + 1) T / P)) of its T tiles, so ragged lengths stay
 *           balanced.  The part of a unit inside one CTA's share is a piece; the CTA that
 *           finishes a unit's last piece merges the pieces by their log-sum-exp (one launch).
 *   workspace: at least attn_decode_workspace_bytes(B, Hq, Hkv, Nq, Nk, d, num_ctas) bytes,
 *           16-byte aligned, and ZEROED before its first use (e.g. cudaMemsetAsync): it holds
 *           one arrival counter per (batch, kv head) at its start, which every completed call
 *           leaves at zero again, so one zeroed workspace of the largest size needed serves
 *           calls with any num_ctas.  After a call that ends in ATTN_ERR_TIMEOUT, zero it again.
 *   kv_lens must be 4-byte aligned; every other pointer 16-byte aligned.
 */
size_t attn_decode_workspace_bytes(int B, int Hq, int Hkv, int Nq, int Nk, int d, int num_ctas);
int attn_decode(const void* q, const void* k_cache, const void* v_cache, const int32_t* kv_lens,
                void* o, float* lse, int B, int Hq, int Hkv, int Nq, int Nk, int d, int causal,
                float scale, int dtype, int num_ctas, void* workspace, size_t ws_bytes,
                void* stream);

/*
 * attn_check_status - synchronises the current device, returns ATTN_OK or
 * ATTN_ERR_TIMEOUT if a device-side wait ran out since the last call, and
 * clears the status word.
 */
int attn_check_status(void);

/*
 * attn_merge_lse - joins two attention results over disjoint key sets by their log-sum-exp, the
 * step a sequence-parallel (ring) attention takes after each exchange.  The "FlashAttention"
 * glossary (deep-dive section, FAQ) rescales partial softmax results by running maxima and sums;
 * for results (O_a, lse_a) and (O_b, lse_b) over key sets A and B the result over A u B is
 *     lse = ln(exp(lse_a) + exp(lse_b)),  O = exp(lse_a - lse) O_a + exp(lse_b - lse) O_b,
 * which is what ring attention (named by the APB article as the exact sequence-parallel
 * baseline) computes after each step.  Float32 arithmetic, one pass over HBM.
 *
 *   rows    number of query rows (B * Hq * Nq); each row holds d values (d = 64 or 128).
 *   o_acc   [rows, d] float32, lse_acc [rows] float32: the running result (device, read and
 *           written).  A row whose lse is -inf has no keys: its O must be 0; it adds no weight.
 *   o_part  [rows, d] 16-bit (dtype), lse_part [rows] float32: one step's result, e.g. the o and
 *           lse outputs of attn_fwd for the same rows (natural-log lse).  Both NULL: nothing is
 *           merged (use with o_out to convert the running result).
 *   first   1: o_acc / lse_acc are set to the part (their contents are ignored); 0: merged.
 *   o_out   [rows, d] 16-bit (dtype) or NULL: receives the merged O rounded to nearest even.
 *   All pointers device, 16-byte aligned; rows = 0 launches nothing.  Errors: ATTN_ERR_ARG
 *   (null accumulator, first without a part, only one of o_part / lse_part, bad dtype or
 *   first), ATTN_ERR_UNSUPPORTED (d), ATTN_ERR_ALIGN.
 */
int attn_merge_lse(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part,
                   void* o_out, long long rows, int d, int dtype, int first, void* stream);

/*
 * attn_test_host_pieces - test hook: the pieces attn_fwd_host cuts the B*Hq query heads into, as
 * cut points cuts[0] = 0 < cuts[1] < ... < cuts[n] = B*Hq; returns n (at most 16) or a negative
 * ATTN_ERR_* code (the shape checks of attn_fwd; cuts NULL or max_cuts < 17 is ATTN_ERR_ARG).
 * Host only: nothing is launched.
 */
int attn_test_host_pieces(int B, int Hq, int Hkv, int N, int d, int* cuts, int max_cuts);

/*
 * attn_test_wait_timeout - test hook for failure detection.  Launches one tiny kernel whose single
 * thread waits on an mbarrier that nothing ever completes, with a limit of `limit_us`
 * microseconds (1..1000000).  The wait gives up, sets the device status word and the kernel
 * returns normally, so the next attn_check_status() returns ATTN_ERR_TIMEOUT and the context
 * stays usable.  No fault, trap or hang is involved.
 */
int attn_test_wait_timeout(int limit_us, void* stream);

/*
 * attn_test_exp2 - test hook: y[i] = 2^x[i] computed by one of the two exp2 routines the fused
 * kernel's softmax uses: use_poly = 1 -> the FMA-pipe routine (range reduction to [-1/2, 1/2]
 * plus a degree-3 minimax polynomial, relative error <= 7.5e-5 for -125 <= x <= 8; inputs below
 * -125 return 2^-125), use_poly = 2 -> the same routine on packed pairs (f32x2 arithmetic; must
 * equal use_poly = 1 bit for bit), use_poly = 0 -> the MUFU ex2.approx instruction.  x, y:
 * device float32 arrays of n >= 1 elements.
 */
int attn_test_exp2(const float* x, float* y, int n, int use_poly, void* stream);

/* Static, human-readable text for an ATTN_* code. */
const char* attn_error_string(int code);

/* The last CUDA error text seen by the library on this thread ("" if none). */
const char* attn_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* TILED_ATTENTION_H */
