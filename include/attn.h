/*
 * C ABI of the B200 (sm_100a) causal prefill attention library, libattn_b200.so.
 *
 * The operation ([ZYFA-fr] = ai-daily-news.org article
 * "zyphra-zyfa-fp8-flashattention-amd-mi355x", section "Ce que couvrent les noyaux";
 * [ZYFA-pt] = acheiumaia.com.br news item "zyphra-zyfa-flashattention-fp8-para-amd-mi355x",
 * TL;DR; [ZYFA-mb] = miraibroadcast.com, "Zyphra lança ZYFA e acelera GPUs AMD em até
 * 1,76x IA", sections "Como o motor de atenção FP8 da Zyphra funciona" and "Precisão,
 * estabilidade e efeito na prática"):
 *
 *   forward causal (prefill) attention  O = softmax(mask(Q K^T * scale)) V
 *   in BF16 or FP8 e4m3, head dim 128 with grouped-query heads, or the MLA shape
 *   (qk dim 192, v dim 128).  The FP8 path forms probabilities with the exp-free lean-P
 *   encoding, scales each 64-key block by a power of two removed by the block-scaled MMA,
 *   and takes the row normaliser from the tensor-core sum of the rounded probabilities.
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers unless stated; the caller allocates and
 *     frees them.  The library never allocates device memory (TMEM is allocated and
 *     released inside each kernel).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are asynchronous
 *     and stream-ordered; they do not synchronise.  They are thread-safe and reentrant.
 *   - Layouts: token-major BSHD, i.e. [B, S, H, d] contiguous with d innermost.
 *   - Synchronous argument checks return an error code before anything is launched; no
 *     exception crosses the ABI.  Kernels never trap: a bounded wait that expires sets a
 *     device error word, reported by attn_device_status().
 *   - Scale = 1/sqrt(d_qk).  Query head h reads key/value head h / (Hq / Hkv).
 *     Causal: key j is visible from query i iff j <= i (Sq == Sk == S).
 */
#ifndef ATTN_B200_H
#define ATTN_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum attn_status {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = 1, /* null pointer, negative size, Hq % Hkv != 0, bad flag */
  ATTN_ERR_UNSUPPORTED = 2, /* head dims other than 128/192 (qk) and 128 (v); a flag or
                               the dump combined with sequences not a multiple of 128 */
  ATTN_ERR_ALIGNMENT = 3,   /* a tensor pointer not 16-byte aligned */
  ATTN_ERR_CUDA = 4,        /* a CUDA runtime call or kernel launch failed */
  ATTN_ERR_TIMEOUT = 5      /* a device-side bounded wait expired (see attn_device_status) */
} attn_status_t;

typedef enum attn_dtype { ATTN_BF16 = 0, ATTN_FP8_E4M3 = 1 } attn_dtype_t;

/* flags of attn_fwd_ex */
#define ATTN_FLAG_UNROTATE_O 1u /* V was Hadamard-rotated: apply x H/sqrt(128) to O rows */
/*
 * FP8 only (else ATTN_ERR_INVALID_ARG): the exact-P ablation that [ZYFA-mb] ("Como o motor
 * de atenção FP8 da Zyphra funciona") contrasts with lean P.  Each probability is formed
 * by an exponential, P = e4m3_rn(2^x) with x = fmaf(s, a/8, (8 (7 + k_b) - m)/8), instead
 * of the lean-P multiply-add and integer conversion; the reference max m, the 64-key block
 * shifts k_b, the block-scaled PV and the row sum are the same.  2^x is evaluated by the
 * hardware approximate exponential (relative error below 2^-21), so codes can differ by
 * one from the correctly rounded e4m3 of 2^x where 2^x lies that close to a rounding
 * midpoint.
 */
#define ATTN_FLAG_EXACT_P 2u

/*
 * attn_fwd: forward causal prefill attention.
 *   q         [B, S, Hq,  d_qk]  bf16 (ATTN_BF16) or e4m3 codes (ATTN_FP8_E4M3)
 *   k         [B, S, Hkv, d_qk]  same type as q
 *   v         [B, S, Hkv, d_v ]  same type as q
 *   o         [B, S, Hq,  d_v ]  bf16 output (round to nearest even)
 *   lse       [B, Hq, S] fp32 natural-log sum-exp of the scaled scores, or NULL
 *   d_qk      128 or 192;  d_v  128
 *   dtype     ATTN_BF16 or ATTN_FP8_E4M3
 *   descale_q/k/v  DEVICE pointers to one fp32 each (x = code * descale), as written by
 *             attn_quantize_e4m3; required for FP8, ignored (may be NULL) for BF16
 *   causal    1 = causal mask (the contract), 0 = full attention
 * Requirements: Hq % Hkv == 0, pointers 16-byte aligned.  Any S >= 0: when S % 128 != 0
 * the kernel variant that masks the keys past the end of each sequence and does not write
 * the rows past it runs (then ATTN_FLAG_EXACT_P is not supported).  B == 0 or S == 0 is a
 * no-op.
 */
attn_status_t attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                       int Hq, int Hkv, int S, int d_qk, int d_v, attn_dtype_t dtype,
                       const float* descale_q, const float* descale_k, const float* descale_v,
                       int causal, void* stream);

/* attn_fwd with option flags (ATTN_FLAG_*). */
attn_status_t attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse,
                          int B, int Hq, int Hkv, int S, int d_qk, int d_v, attn_dtype_t dtype,
                          const float* descale_q, const float* descale_k,
                          const float* descale_v, int causal, unsigned flags, void* stream);

/*
 * attn_fwd_varlen: attn_fwd over a batch of sequences of different lengths packed along
 * the token axis (variable-length batches, which [ZYFA-fr] "Ce que couvrent les noyaux"
 * lists as not yet supported by the pages' kernels).
 *   q [T, Hq, d_qk], k [T, Hkv, d_qk], v [T, Hkv, d_v], o [T, Hq, d_v] (T = total_tokens),
 *   same types and head rules as attn_fwd; lse [Hq, T] fp32 or NULL.
 *   cu_seqlens  DEVICE int32 [B + 1]: sequence b is tokens [cu_seqlens[b], cu_seqlens[b+1]);
 *               non-decreasing, cu_seqlens[0] >= 0, cu_seqlens[B] <= T, each length at
 *               most max_seqlen.  Read by the kernel (no host synchronisation): a sequence
 *               that breaks these rules is skipped (its outputs are not written) and
 *               attn_device_status() then reports ATTN_ERR_INVALID_ARG.
 *   max_seqlen  the longest sequence (sizes the grid), <= T.
 *   causal      1: key j of a sequence is visible from its query i iff j <= i.
 *   flags       ATTN_FLAG_UNROTATE_O only (ATTN_FLAG_EXACT_P: ATTN_ERR_UNSUPPORTED).
 * Tokens not covered by any sequence are not written.  B == 0, max_seqlen == 0 or T == 0 is
 * a no-op.  Requirements: pointers 16-byte aligned (cu_seqlens 4-byte), T <= 2^31 - 1.
 */
attn_status_t attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                              const int32_t* cu_seqlens, int B, int max_seqlen,
                              int64_t total_tokens, int Hq, int Hkv, int d_qk, int d_v,
                              attn_dtype_t dtype, const float* descale_q, const float* descale_k,
                              const float* descale_v, int causal, unsigned flags, void* stream);

/*
 * attn_decode_paged: decode attention over a paged KV cache -- one new query token per
 * sequence against every cached token of its sequence, the cache holding the token itself
 * (decode and paged KV caches are listed as not yet supported by the pages' kernels,
 * [ZYFA-fr] "Ce que couvrent les noyaux").
 *   q          [B, Hq, 128]  bf16, or e4m3 codes (ATTN_FP8_E4M3) with descale_q
 *   k_cache    [num_pages, page_size, Hkv, 128]  same type as q (FP8: descale_k)
 *   v_cache    [num_pages, page_size, Hkv, 128]  same type (FP8: descale_v)
 *   o          [B, Hq, 128] bf16;  lse [B, Hq] fp32 natural log, or NULL
 *   block_table DEVICE int32 [B, max_blocks_per_seq]: token j of sequence b is slot
 *              j % page_size of page block_table[b][j / page_size]
 *   seq_lens   DEVICE int32 [B]: cached tokens of each sequence, <= max_seqlen
 *   max_seqlen the longest sequence (sizes the split of the work), <= max_blocks_per_seq *
 *              page_size
 *   workspace  DEVICE scratch of at least attn_decode_workspace_size(B, Hq, Hkv, max_seqlen)
 *              bytes (16-byte aligned), owned by the caller; not shared by concurrent calls
 * o = softmax(q K^T / sqrt(128)) V over the sequence's tokens; query head h reads kv head
 * h / (Hq / Hkv).  A sequence of length 0 gives o = 0, lse = -inf.  Lengths and page ids
 * are read on the device: a length above max_seqlen or a page id outside [0, num_pages)
 * skips that (sequence, kv head) range and attn_device_status() reports
 * ATTN_ERR_INVALID_ARG; nothing outside the cache is read.  Computed in fp32.
 * Requirements: d_qk = d_v = 128; Hq / Hkv in {1, 2, 4, 8, 16}; page_size a power of two
 * <= 65536; caches and workspace 16-byte aligned.  B == 0 is a no-op.
 */
attn_status_t attn_decode_paged(const void* q, const void* k_cache, const void* v_cache, void* o,
                                float* lse, const int32_t* block_table, const int32_t* seq_lens,
                                int B, int Hq, int Hkv, int d_qk, int d_v, int num_pages,
                                int page_size, int max_blocks_per_seq, int max_seqlen,
                                attn_dtype_t dtype, const float* descale_q,
                                const float* descale_k, const float* descale_v, void* workspace,
                                size_t workspace_bytes, void* stream);
size_t attn_decode_workspace_size(int B, int Hq, int Hkv, int max_seqlen);

/*
 * attn_quantize_e4m3: per-tensor e4m3 quantisation of a bf16 tensor [tokens, H, d]
 * ([ZYFA-mb], "Precisão, estabilidade e efeito na prática").
 *   y = x, or with hadamard = 1, y = (x H_128) * float32(1/sqrt(128)) along d (d must be
 *   128), computed in float32 by butterfly stages h = 1, 2, ..., 64;
 *   amax = max|y|; scale = 448/amax; codes = e4m3 round-to-nearest-even, saturating, of
 *   float32(y * scale); *descale_out = amax/448 (both 1 when amax == 0).
 *   x_bf16     device, [tokens, H, d] bf16, 16-byte aligned
 *   x_e4m3     device, [tokens, H, d] uint8 output, 16-byte aligned
 *   descale_out device, one fp32
 *   workspace  device scratch of at least attn_quantize_workspace_size() bytes, 4-byte
 *              aligned, owned by the caller; must not be shared by calls running
 *              concurrently
 * Requirements: d % 8 == 0.  Deterministic.
 */
attn_status_t attn_quantize_e4m3(const void* x_bf16, void* x_e4m3, float* descale_out,
                                 int64_t tokens, int H, int d, int hadamard, void* workspace,
                                 size_t workspace_bytes, void* stream);
size_t attn_quantize_workspace_size(int64_t tokens, int H, int d);

/*
 * attn_quantize_qkv_e4m3: attn_quantize_e4m3 of Q, K and V of one attention call in two
 * launches (one amax pass and one conversion pass over the three tensors) instead of six;
 * codes and descales identical to three attn_quantize_e4m3 calls.
 *   q, k, v      device bf16 [tokens, Hq, d_qk], [tokens, Hkv, d_qk], [tokens, Hkv, d_v]
 *   q8, k8, v8   device uint8 outputs of the same shapes; descale_q/k/v one fp32 each
 *   hadamard     0, or 1 to rotate all three (d_qk = d_v = 128)
 *   workspace    device scratch of at least attn_quantize_qkv_workspace_size() bytes,
 *                4-byte aligned, not shared by calls running concurrently
 * Requirements: d_qk % 8 == d_v % 8 == 0, tensors 16-byte aligned.  tokens == 0 sets the
 * three descales to 1.
 */
attn_status_t attn_quantize_qkv_e4m3(const void* q, const void* k, const void* v, void* q8,
                                     void* k8, void* v8, float* descale_q, float* descale_k,
                                     float* descale_v, int64_t tokens, int Hq, int Hkv, int d_qk,
                                     int d_v, int hadamard, void* workspace,
                                     size_t workspace_bytes, void* stream);
size_t attn_quantize_qkv_workspace_size(void);

/*
 * attn_quantize_e4m3_static: attn_quantize_e4m3 for callers that cannot allocate device
 * memory (e.g. a plugin inside an engine that owns and pre-plans all device memory, or a
 * latency-critical loop where cudaMalloc's possible device synchronisation is not allowed).
 * The pages have no counterpart: it is an interface convenience of this library.
 *   Same arguments, results and codes as attn_quantize_e4m3, minus the workspace: the
 *   scratch is a fixed 256-byte array compiled into the library, held on every GPU that
 *   loads it until the process exits.  A problem whose scratch need
 *   (attn_quantize_workspace_size) exceeds 256 bytes returns ATTN_ERR_UNSUPPORTED.
 *   Every call looks up the array's device address in the current context (a lookup that
 *   allocates nothing), so the address stays valid after cudaDeviceReset or with a
 *   non-primary context.  The first call on a device may load the library's device code on
 *   it: make that first call before any stream capture.  All calls share the array (it
 *   keeps the last call's contents; the amax word is cleared at the start of each call), so
 *   calls that may overlap on the GPU -- on different streams, or from different host
 *   threads -- race and must be serialised by the caller.  Allocates nothing.
 */
attn_status_t attn_quantize_e4m3_static(const void* x_bf16, void* x_e4m3, float* descale_out,
                                        int64_t tokens, int H, int d, int hadamard,
                                        void* stream);

/*
 * Test-only: FP8 attn_fwd_ex that also dumps, for every (query row, visible key tile), the
 * raw fp32 scores after masking, the P e4m3 codes (lean P, or exact P with
 * ATTN_FLAG_EXACT_P in flags) and the per-64-key shifts:
 *   dump_s      [B, Hq, S, S] fp32      dump_codes [B, Hq, S, S] uint8
 *   dump_kshift [B, Hq, S, S/64] uint8  (entries of key tiles that are not visible are
 *   left untouched).  d_qk must be 128 or 192; slow; for small S only.
 */
attn_status_t attn_fwd_fp8_dump(const void* q, const void* k, const void* v, void* o, float* lse,
                                int B, int Hq, int Hkv, int S, int d_qk, int d_v,
                                const float* descale_q, const float* descale_k,
                                const float* descale_v, int causal, unsigned flags,
                                float* dump_s, uint8_t* dump_codes, uint8_t* dump_kshift,
                                void* stream);

/*
 * Synchronises `stream` and reports (then clears) the device error word of the current
 * device: ATTN_ERR_TIMEOUT if a kernel's bounded wait expired, ATTN_ERR_CUDA if the stream
 * reported an error, ATTN_OK otherwise.
 */
attn_status_t attn_device_status(void* stream);

/*
 * Work unit and schedule of the prefill kernel used by attn_fwd, attn_fwd_ex,
 * attn_fwd_varlen and the dump: the bitwise OR of a unit (a CTA's two 128-row query slots
 * in ping-pong sharing every K/V tile) and at most one schedule flag:
 *   ATTN_KERNEL_SINGLE      (0) two consecutive query tiles of one query head;
 *   ATTN_KERNEL_HEADS       (2) one query tile of two query heads of one kv group (equal
 *                           causal extents); with Hq / Hkv odd it is ATTN_KERNEL_SINGLE;
 *   ATTN_KERNEL_PERSISTENT  (4) one CTA per SM, each running a static list of units
 *                           (rounds of SM-count units, alternate rounds mirrored);
 *   ATTN_KERNEL_DYNAMIC     (8) one CTA launched per unit (longest first); a CTA that
 *                           finishes its unit takes over the unit of a CTA that has not
 *                           started yet (cluster launch control), so each SM keeps one CTA
 *                           running unit after unit.
 * Without a schedule flag every CTA runs one unit.  For BF16, at most one pipeline flag:
 *   ATTN_KERNEL_BF16_S_AHEAD  (32) the pipeline of the FP8 kernel: one warp issues S_t(j+1)
 *                             as soon as both slots have read their latest S (the two
 *                             slots alternate in one S buffer in TMEM), another PV_t(j)
 *                             from P_t in TMEM columns of its own;
 *   ATTN_KERNEL_BF16_P_OVER_S (64) P_t written over the S_t columns it came from, one warp
 *                             issuing PV_t(j) then S_t(j+1).
 * Without one (and with ATTN_KERNEL_AUTO) BF16 uses S-ahead when Hq > Hkv, P-over-S when
 * Hq == Hkv (measured faster there: with a kv head per query head the K/V tiles stream from
 * HBM and S-ahead needs them earlier).  FP8 ignores the pipeline flags.  ATTN_KERNEL_AUTO
 * (16, alone; the default) is ATTN_KERNEL_DYNAMIC with head pairs for FP8 and tile pairs
 * for BF16.  All compute the same function (bitwise the same outputs and lean-P codes: a
 * unit is computed by the same code whichever CTA runs it, and both BF16 pipelines issue the
 * same MMAs in the same order per slot).  A process-wide setting, for measurement and tests;
 * returns ATTN_ERR_INVALID_ARG for another value.
 */
#define ATTN_KERNEL_SINGLE 0
#define ATTN_KERNEL_HEADS 2
#define ATTN_KERNEL_PERSISTENT 4
#define ATTN_KERNEL_DYNAMIC 8
#define ATTN_KERNEL_AUTO 16
#define ATTN_KERNEL_BF16_S_AHEAD 32
#define ATTN_KERNEL_BF16_P_OVER_S 64
attn_status_t attn_select_prefill_kernel(int kernel);

/* Test-only: sets the bounded-wait limit in nanoseconds (0 restores the default, 2 s). */
void attn_set_wait_timeout_ns(uint64_t ns);

/*
 * Test-only: the prefill kernels' load warp stops before key tile `tile` (a negative value
 * restores normal operation), so the waits on that tile are never satisfied: they run out
 * after the bounded-wait limit, the kernel records ATTN_ERR_TIMEOUT in the device error word
 * and every warp unwinds (no copy or MMA is left in flight), leaving the context usable.
 * Applies to the attn_fwd* calls made while it is set.
 */
void attn_selftest_stall_tile(int tile);

/*
 * Test-only: caps the grid of the persistent schedule (ATTN_KERNEL_PERSISTENT) at n CTAs, so
 * that small problems run many units per CTA (n <= 0 removes the cap).
 */
void attn_selftest_max_ctas(int n);

/*
 * Test-only: launches one thread that waits, with the bounded wait the kernels use, on an
 * mbarrier that nothing completes.  The wait gives up after timeout_ns (1 ns .. 10 s) and
 * records the timeout in the device error word, so attn_device_status() then reports
 * ATTN_ERR_TIMEOUT and the context stays usable.
 */
attn_status_t attn_selftest_wait_timeout(uint64_t timeout_ns, void* stream);

const char* attn_status_string(attn_status_t status);
int attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_H */
