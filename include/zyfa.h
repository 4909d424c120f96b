/*
 * zyfa.h -- C ABI of libzyfa.so: causal prefill attention forward for NVIDIA
 * B200 (sm_100a) with FP8 e4m3 or BF16 Q/K/V, following Zyphra's ZYFA method
 * (Lean-P FP8 probabilities, a power-of-two scale per 64-key block, the row sum
 * taken from the rounded probabilities), plus its quantize + Hadamard prepass.
 *
 * Sources (news pages about ZYFA):
 *   the-ai.news, "Zyphra presenteert ZYFA: FlashAttention FP8 voor AMD MI355X"
 *   ai-daily-news.org, "Zyphra ZYFA: FP8 FlashAttention para AMD MI355X"
 *   kongchang.com, "Zyphra ZYFA: AMD MI355X 上的 FP8 FlashAttention 提速 1.76 倍"
 *   spke.com, "Zyphra ZYFA: AMD MI355X向けFP8 FlashAttention、最大1.76倍高速化"
 *
 * Conventions for every entry point:
 *  - Pointers named q, k, v, o, lse, x, x_fp8, scale, *_scale and the Lean-P
 *    test arrays are DEVICE pointers (CUDA global memory of the current
 *    device); cu_seqlens and the schedule query's units are HOST arrays.
 *    The caller allocates and owns every buffer; the library allocates no
 *    memory and keeps no state between calls other than one device error
 *    word (see zyfa_device_status) and per-device launch attributes.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Work is
 *    enqueued asynchronously on it; no other stream is used.
 *  - Return value: ZYFA_OK (0) once the work is enqueued, or a negative
 *    zyfa_status.  On any argument error nothing is launched.  Faults inside
 *    a kernel surface at the caller's next synchronisation; bounded waits that
 *    run out inside the attention kernel are reported by zyfa_device_status.
 *  - Layouts are BSHD, contiguous, innermost dimension last (the
 *    flash_attn_func convention that the pages' drop-in Python interface
 *    uses: spke.com "Zyphra ZYFA", TL;DR).
 *  - All calls are reentrant; results are deterministic (fixed ascending
 *    key-tile order, no atomics on data; the pages report bitwise identical
 *    output across 7,200 runs: spke.com "Zyphra ZYFA", accuracy section).
 */
#ifndef ZYFA_H_
#define ZYFA_H_

#ifdef __cplusplus
extern "C" {
#endif

/* Element types. */
enum zyfa_dtype {
  ZYFA_BF16 = 0,      /* bfloat16 */
  ZYFA_FP8_E4M3 = 1,  /* OCP e4m3 "fn": bias 7, max 448, 0x7F/0xFF NaN */
  ZYFA_FP32 = 2       /* IEEE binary32 (prepass input only) */
};

/* Status codes (negative = error). */
enum zyfa_status {
  ZYFA_OK = 0,
  ZYFA_ERR_NULL_PTR = -1,            /* a required pointer is NULL */
  ZYFA_ERR_BAD_SHAPE = -2,           /* B, S, H < 1, or sizes overflow the TMA index range */
  ZYFA_ERR_UNSUPPORTED_HEADDIM = -3, /* (Dqk, Dv) not (128,128) or (192,128); prepass D */
  ZYFA_ERR_BAD_GQA = -4,             /* Hq is not a multiple of Hkv */
  ZYFA_ERR_MISALIGNED = -5,          /* a tensor base is not 16-byte aligned (scales: 4) */
  ZYFA_ERR_BAD_DTYPE = -6,           /* dtype / in_dtype / flag value not supported */
  ZYFA_ERR_CUDA = -7,                /* a CUDA runtime/driver call or launch failed */
  ZYFA_ERR_DEVICE_TIMEOUT = -8       /* a bounded device wait ran out (zyfa_device_status) */
};

/*
 * zyfa_attn_fwd -- causal prefill attention forward (prefill only, Sq = Sk):
 *
 *     O = softmax(Q K^T / sqrt(Dqk) + causal mask) V
 *
 * The computation the pages describe (ai-daily-news.org "Zyphra ZYFA",
 * "Qué cubren los kernels": causal forward attention in FP8 and BF16, head
 * dimension 128 and DeepSeek-V2's latent-attention shape; spke.com TL;DR:
 * MLA shape 192/128).
 *
 *   q  [B, S, Hq,  Dqk]   dtype elements
 *   k  [B, S, Hkv, Dqk]   dtype elements
 *   v  [B, S, Hkv, Dv ]   dtype elements
 *   o  [B, S, Hq,  Dv ]   bfloat16 output (written for every row < S)
 *   Query head h reads kv head h / (Hq / Hkv) (grouped-query attention).
 *   (Dqk, Dv) in {(128, 128), (192, 128)}; S >= 1; B, Hq, Hkv >= 1.
 *   Softmax scale is fixed at 1/sqrt(Dqk).
 *
 * dtype = ZYFA_BF16: exact softmax probabilities (exp2, fp32), P rounded to
 *   bf16 for the P V product; the row sum is accumulated in fp32 from the
 *   unrounded probabilities.  Scale pointers are ignored.
 * dtype = ZYFA_FP8_E4M3: q/k/v hold e4m3 codes; the real values are
 *   code * scale with one fp32 scale per (batch, head):
 *     q_scale [B*Hq], k_scale [B*Hkv], v_scale [B*Hkv]  (device; NULL = 1.0),
 *   indexed b*H + h.  P is written Lean-P style (the-ai.news "Zyphra presenteert
 *   ZYFA", "Drie technieken om de bottleneck te omzeilen"; spke.com "Lean P"):
 *   one multiply-add and one integer conversion per probability, code of 2^x
 *   ~ 8x + 56, truncated, with a power-of-two 2^j per (row, 64-key block)
 *   applied before rounding and removed by the block-scaled tensor-core MMA
 *   (spke.com "ブロックごとのスケーリングと丸められた行和").  The softmax
 *   denominator is the sum of the rounded, rescaled probabilities, taken by an
 *   extra MMA against a ones matrix.  Accumulation is fp32 throughout.
 *
 * Alignment: q, k, v, o 16-byte aligned; scales 4-byte aligned.
 * Errors: NULL_PTR (q, k, v or o NULL), BAD_SHAPE, BAD_GQA,
 *   UNSUPPORTED_HEADDIM, BAD_DTYPE, MISALIGNED, CUDA.
 */
int zyfa_attn_fwd(const void* q, const void* k, const void* v, void* o, int B, int Hq, int Hkv,
                  int S, int Dqk, int Dv, int dtype, const float* q_scale, const float* k_scale,
                  const float* v_scale, void* stream);

/*
 * zyfa_attn_fwd_lse -- zyfa_attn_fwd plus each row's softmax log-sum-exp, for
 * callers that combine partial attention results (the online softmax of
 * kongchang.com "Zyphra ZYFA", FlashAttention tiling, keeps exactly the
 * running max and row sum this is formed from):
 *   lse [B, Hq, S] fp32 (caller-owned, 4-byte aligned), natural log of
 *   sum over keys j <= i of exp(s_ij / sqrt(Dqk)), s_ij the dot product of
 *   the values the kernel received (dequantized for FP8).  It is formed from
 *   the kernel's final reference max m and row sum l: ln 2 (m c + log2 l)
 *   with c = log2(e) q_s k_s / sqrt(Dqk); for FP8, l sums the rounded Lean-P
 *   weights, so the FP8 value carries their error (a few 1e-2 absolute).
 * Other arguments, layouts and errors as zyfa_attn_fwd; NULL lse is
 * ZYFA_ERR_NULL_PTR.
 */
int zyfa_attn_fwd_lse(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                      int Hkv, int S, int Dqk, int Dv, int dtype, const float* q_scale,
                      const float* k_scale, const float* v_scale, void* stream);

/*
 * zyfa_attn_fwd_fp8_exact_p -- the exact-P ablation of the FP8 path: the
 * pages' Lean P (the-ai.news "Zyphra presenteert ZYFA", section "Drie
 * technieken om de bottleneck te omzeilen"; spke.com "Zyphra ZYFA", section
 * "Lean P") replaces the conventional way of writing P in FP8, an
 * exponential followed by a conversion to e4m3.  This entry runs that
 * conventional way in the same kernel: each probability is
 * e4m3 RNE-satfinite of ex2((s - m) A / 8 + j), with the same deferred
 * reference max, the same 64-key block shift j and E8M0 scales, and the same
 * row sum over the rounded P, so the two can be compared on speed and error.
 * Arguments, layouts, ownership and errors as zyfa_attn_fwd with
 * dtype = ZYFA_FP8_E4M3.
 */
int zyfa_attn_fwd_fp8_exact_p(const void* q, const void* k, const void* v, void* o, int B, int Hq,
                              int Hkv, int S, int Dqk, int Dv, const float* q_scale,
                              const float* k_scale, const float* v_scale, void* stream);

/*
 * zyfa_quantize -- the prepass: per-(batch, head) FP8 e4m3 quantization, with
 * an optional Hadamard rotation for Q and K (spke.com "Zyphra ZYFA", accuracy
 * section: most FP8 error comes from quantizing Q, K and V, and a Hadamard
 * rotation of Q and K roughly halves it; kongchang.com "ZYFA 的性能与精度数据":
 * per-tensor or per-head scale factors map values into the e4m3 range).
 *
 *   x      [B, S, H, D]  in_dtype = ZYFA_BF16 or ZYFA_FP32
 *   x_fp8  [B, S, H, D]  e4m3 codes (output)
 *   scale  [B*H]         fp32 (output), indexed b*H + h
 *   hadamard = 1: each D = 128 row is first rotated by the orthonormal
 *     128-point Sylvester Walsh-Hadamard transform (butterflies of stride
 *     1, 2, ..., 64 in fp32, then one multiply by fp32(2^-3.5)).  A D = 192
 *     row (the MLA shape) is rotated block-diagonally: dims 0..127 by that
 *     transform, dims 128..191 by the 64-point one (strides 1 .. 32, then
 *     times 2^-3).  Apply it to Q and K only (the rotation cancels in Q K^T);
 *     never to V.
 *   For each (b, h): amax = max |x'| over (s, d); scale = amax / 448 (fp32,
 *   IEEE division; 1.0 when amax == 0); code = e4m3 round-to-nearest-even,
 *   saturating at +-448, of fp32(x' / scale) (IEEE division).
 * D must be a multiple of 8 and at most 1024 (128 or 192 with hadamard).
 * Alignment: x and x_fp8 16-byte aligned; scale 4-byte aligned.  The scale
 * buffer is used as the amax accumulator while the prepass runs (four
 * stream-ordered steps); it holds the final scales once the stream reaches
 * the end of the call.
 */
int zyfa_quantize(const void* x, int in_dtype, void* x_fp8, float* scale, int B, int S, int H,
                  int D, int hadamard, void* stream);

/*
 * zyfa_quantize_qkv -- the same prepass for Q, K and V at once (the sources
 * above): byte for byte the result of
 *   zyfa_quantize(q, in_dtype, q_fp8, q_scale, B, S, Hq, Dqk, hadamard_qk, s)
 *   zyfa_quantize(k, in_dtype, k_fp8, k_scale, B, S, Hkv, Dqk, hadamard_qk, s)
 *   zyfa_quantize(v, in_dtype, v_fp8, v_scale, B, S, Hkv, Dv, 0, s)
 * in four kernel launches instead of twelve (each step of the prepass runs
 * over the three tensors in one grid, shared in proportion to their bytes).
 *   q [B, S, Hq, Dqk], k [B, S, Hkv, Dqk], v [B, S, Hkv, Dv]: in_dtype
 *   *_fp8: e4m3 codes of the same shapes (outputs, caller-owned)
 *   *_scale: fp32 [B*Hq], [B*Hkv], [B*Hkv] (outputs; used as amax
 *   accumulators while the call's kernels run)
 * Dqk and Dv: multiples of 8, at most 1024 (Dqk = 128 or 192 with hadamard_qk = 1).
 * Alignment as for zyfa_quantize.  Errors as for zyfa_quantize; nothing is
 * launched when an argument is rejected.
 */
int zyfa_quantize_qkv(const void* q, const void* k, const void* v, int in_dtype, void* q_fp8,
                      void* k_fp8, void* v_fp8, float* q_scale, float* k_scale, float* v_scale,
                      int B, int S, int Hq, int Hkv, int Dqk, int Dv, int hadamard_qk, void* stream);

/*
 * Variable-length batches.  The pages list them as future work for the
 * method (ai-daily-news.org "Zyphra ZYFA", "Qué cubren los kernels": no
 * decode, no paged KV caches, no variable-length batches); these entries
 * extend the same computation to a packed batch of independent sequences.
 *
 * Packing: sequence s (0 <= s < nseq) holds rows cu_seqlens[s] ..
 * cu_seqlens[s+1]-1 of every tensor; T = cu_seqlens[nseq] rows in all.
 * cu_seqlens is a HOST array of nseq + 1 ints (read during the call, not
 * kept): cu_seqlens[0] = 0, non-decreasing (empty sequences allowed).
 * 1 <= nseq <= 384 per call.  Every sequence is causal on its own: row i of
 * sequence s attends to rows 0..i of s only, and its output does not depend
 * on the other sequences of the batch (FP8: each sequence has its own
 * scales).  Precondition: the inputs are finite (a non-finite value could
 * reach a neighbouring sequence through a masked, zero weight).
 */

/*
 * zyfa_attn_fwd_varlen -- zyfa_attn_fwd over a packed batch.
 *   q  [T, Hq,  Dqk], k [T, Hkv, Dqk], v [T, Hkv, Dv]   dtype elements
 *   o  [T, Hq,  Dv ]  bfloat16 (every row of every sequence written)
 *   lse [Hq, T] fp32, or NULL: each row's log-sum-exp as in zyfa_attn_fwd_lse
 *   q_scale [nseq*Hq], k_scale [nseq*Hkv], v_scale [nseq*Hkv] (FP8; device;
 *     NULL = 1.0), indexed s*H + h: one scale per (sequence, head).
 * Each row's output is bit-identical to zyfa_attn_fwd (B = 1) on its
 * sequence alone.  Scheduling: sequences longest first, heaviest query tiles
 * first, K/V of a group of (sequence, kv head) slots kept in L2.
 * Errors: NULL_PTR (a tensor or cu_seqlens NULL), BAD_SHAPE (nseq out of
 * range, cu_seqlens not as above), BAD_GQA, UNSUPPORTED_HEADDIM, BAD_DTYPE,
 * MISALIGNED (tensors 16-byte, scales and lse 4-byte), CUDA.  T = 0 is valid
 * and launches nothing (the tensor pointers may then be NULL).  The library
 * cannot see tensor sizes: each tensor must hold T rows.
 */
int zyfa_attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                         const int* cu_seqlens, int nseq, int Hq, int Hkv, int Dqk, int Dv, int dtype,
                         const float* q_scale, const float* k_scale, const float* v_scale, void* stream);

/*
 * zyfa_quantize_varlen -- zyfa_quantize over a packed batch: x and x_fp8
 * [T, H, D], scale [nseq*H] (output), one scale per (sequence, head), so the
 * codes and scale of sequence s equal zyfa_quantize (B = 1) on its rows
 * alone (an empty sequence gets scale 1.0).  Other arguments and errors as
 * zyfa_quantize, plus the cu_seqlens rules above; with T = 0, x and x_fp8
 * may be NULL (only the scales are written).
 */
int zyfa_quantize_varlen(const void* x, int in_dtype, void* x_fp8, float* scale, const int* cu_seqlens,
                         int nseq, int H, int D, int hadamard, void* stream);

/*
 * zyfa_quantize_qkv_varlen -- zyfa_quantize_qkv over a packed batch: byte for
 * byte zyfa_quantize_varlen on Q and K (hadamard_qk) and on V (no rotation),
 * in four launches.  q [T, Hq, Dqk], k [T, Hkv, Dqk], v [T, Hkv, Dv];
 * scales [nseq*Hq], [nseq*Hkv], [nseq*Hkv].
 */
int zyfa_quantize_qkv_varlen(const void* q, const void* k, const void* v, int in_dtype, void* q_fp8,
                             void* k_fp8, void* v_fp8, float* q_scale, float* k_scale, float* v_scale,
                             const int* cu_seqlens, int nseq, int Hq, int Hkv, int Dqk, int Dv,
                             int hadamard_qk, void* stream);

/*
 * zyfa_attn_kv_tile -- host only: the keys per KV tile of the attention
 * kernel that zyfa_attn_fwd (and its _lse, _fp8_exact_p and _varlen forms)
 * runs for this dtype and Dqk: 256 for FP8 with Dqk 128 (S = Q K^T over a
 * 256-key tile is one N = 256 tensor-core accumulator), 128 otherwise.  The
 * deferred reference max of the online softmax (the running max that the
 * probabilities are taken against, which moves only when a tile's max
 * exceeds it by more than 64 binades) is decided once per such tile, so a
 * replay of the FP8 pipeline needs it.  Returns ZYFA_ERR_BAD_DTYPE or
 * ZYFA_ERR_UNSUPPORTED_HEADDIM for arguments zyfa_attn_fwd would reject.
 */
int zyfa_attn_kv_tile(int dtype, int Dqk);

/*
 * zyfa_attn_schedule -- host only (no device call): the work units that CTA
 * `cta` of a `grid`-CTA attention launch processes, in order, as the kernel
 * enumerates them.  A unit is (b, hq, qt): query tile qt (rows 128 qt ..
 * 128 qt + 127) of query head hq of batch entry / sequence b, which takes
 * key tiles 0 .. (128 qt) / kv_tile (kv_tile from zyfa_attn_kv_tile).  Fixed length: cu_seqlens = NULL, B entries of S rows.
 * Packed: cu_seqlens as above with nseq = B (S ignored).  The launch itself
 * uses grid = min(units, SM count).  Writes min(count, cap) units as int
 * triples to `units` (host memory) and returns the count, or a negative
 * status (BAD_SHAPE, BAD_GQA, UNSUPPORTED_HEADDIM, BAD_DTYPE, NULL_PTR).
 */
int zyfa_attn_schedule(int B, int S, const int* cu_seqlens, int Hq, int Hkv, int Dqk, int dtype, int grid,
                       int cta, int* units, int cap);

/* Human-readable text of a status code (static storage; never NULL). */
const char* zyfa_status_string(int status);

/*
 * zyfa_device_status -- synchronises `stream`, then reads and clears the
 * device error word of the current device.  Returns ZYFA_OK, or
 * ZYFA_ERR_DEVICE_TIMEOUT if a bounded wait inside a kernel ran out since the
 * last call (that kernel's output is then invalid), or ZYFA_ERR_CUDA.
 */
int zyfa_device_status(void* stream);

/*
 * zyfa_set_wait_timeout_ns -- time limit of every mbarrier wait inside the
 * attention kernel, in nanoseconds (default 2e9; also read once from the
 * environment variable ZYFA_WAIT_TIMEOUT_MS).  A wait that runs out records
 * ZYFA_ERR_DEVICE_TIMEOUT and the kernel returns without writing the
 * remaining output.  0 restores the default.  Process-wide.
 */
void zyfa_set_wait_timeout_ns(unsigned long long ns);

/*
 * zyfa_device_check -- for a checked build of the library (compiled with
 * ZYFA_CHECKS, libzyfa_checked.so): synchronises `stream`, then reads and
 * clears the range-check word of the current device.  Returns 0 if no check
 * failed since the last call, else the site of the first failure: 1 a
 * scheduled unit's batch, head or tile index; 2 a tile's first row outside
 * its sequence; 3 a scale read outside [B*H]; 4 an output or LSE row outside
 * the tensor (the guarded access was skipped).  ZYFA_ERR_CUDA on a CUDA
 * error.  A normal build never fails a check (it compiles none) and returns 0.
 */
int zyfa_device_check(void* stream);

/* zyfa_checked_build -- 1 for the checked build, 0 for the normal one. */
int zyfa_checked_build(void);

/*
 * zyfa_leanp_codes -- runs the very __device__ functions the FP8 attention
 * kernels use to turn scores into Lean-P codes, so that the codes can be
 * compared byte for byte with a CPU emulation: the per-element steps below,
 * then the same packing of four codes into one 32-bit word (elements
 * 4k .. 4k+3 share a word).  For element i:
 *   j[i]    = 8 if bmax[i] == -inf, else
 *             min(126, 8 + floor(fp32(fp32(m[i] - bmax[i]) * A[i]) * 0.125))
 *   B       = fma(-m[i], A[i], 56 + 8 j[i])
 *   code[i] = masked[i] ? 0 : trunc(max(fma(s[i], A[i], B), 0))   (e4m3 code)
 * (the-ai.news "Zyphra presenteert ZYFA", "Drie technieken ..."; spke.com
 * "Lean P").  Precondition, as inside the kernel: s <= bmax, or s = -inf,
 * and j >= -56.  The kernel's reference max m is deferred (it moves only when
 * a key tile's max exceeds it by more than 64 binades, (tmax - m) A > 512),
 * so bmax may exceed m by up to 512 / A and j then lies in -56..8; a
 * negative j means an E8M0 scale 127 - j above 127 (a weight factor 2^-j
 * above 1).  The block max lands in the top binade (u in (112, 120]) for
 * every j.  Outside the precondition (u >= 127) the device functions do not
 * clamp at 126 and the code is unspecified.
 *   s, m, bmax, A: fp32 [n]; masked: uint8 [n] or NULL; code: uint8 [n];
 *   j: int32 [n] or NULL.  n >= 0.  Errors: NULL_PTR, BAD_SHAPE, CUDA.
 */
int zyfa_leanp_codes(const float* s, const float* m, const float* bmax, const float* A,
                     const unsigned char* masked, int n, unsigned char* code, int* j, void* stream);

/*
 * zyfa_selftest_wait_timeout -- launches a one-CTA kernel whose only thread
 * waits on an mbarrier that nothing ever arrives on, with the given time
 * limit (ns, at most 1e9), through the same bounded-wait routine the attention
 * kernel uses.  The wait runs out, the kernel records ZYFA_ERR_DEVICE_TIMEOUT
 * in the device error word and returns; no fault, trap or hang.  Used to test
 * the failure path: call it, then zyfa_device_status() must report the timeout.
 */
int zyfa_selftest_wait_timeout(unsigned long long timeout_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* ZYFA_H_ */
