/*
 * fa_b200 — exact IO-aware scaled dot-product attention for NVIDIA B200 (sm_100a).
 *
 * The operation (catalogue record "Dao and colleagues: IO-aware exact
 * attention with FlashAttention", field summary; topic page "Flash Attention
 * and Efficient Transformer Mechanisms", opening paragraphs): for every
 * (sequence b, query head h), with key/value head g = h / (Hq / Hkv),
 *
 *     S   = scale * Q[b,:,h,:] K[b,:,g,:]^T      (causal: key j > query i is -inf)
 *     LSE = logsumexp over keys of S              (natural log, per query row)
 *     O   = softmax(S) V[b,:,g,:]
 *
 * computed tile by tile with an online softmax so the N x N score matrix is
 * never written to memory; the backward pass recomputes it from Q, K, V and
 * LSE (the record's summary: recomputation). Nothing is approximated: results
 * differ from the exact value only by floating-point rounding.
 *
 * Conventions shared by every entry point:
 *  - All tensor arguments are DEVICE pointers owned by the caller; the library
 *    never allocates, frees or retains them past the call, and never
 *    synchronises except in fa_get_status().
 *  - Layouts are contiguous, row-major:
 *      padded: Q/O/dO/dQ [B, N, Hq, d], K/V/dK/dV [B, N, Hkv, d]  (BSHD),
 *              LSE [B, Hq, N] float32;
 *      packed (varlen): Q/O [T, Hq, d], K/V [T, Hkv, d], LSE [Hq, T];
 *      sequence s occupies tokens cu_seqlens[s] .. cu_seqlens[s+1]-1.
 *  - bf16 tensors hold __nv_bfloat16 (IEEE bfloat16); fp8 tensors hold
 *    __nv_fp8_e4m3 (OCP e4m3, "fn" variant).
 *  - Data pointers must be 16-byte aligned, LSE 4-byte aligned.
 *  - Supported head dimensions: d = 64 or 128. Hq must be a multiple of Hkv.
 *  - Work is launched asynchronously on `stream` (a cudaStream_t; NULL is the
 *    legacy default stream). Calls are re-entrant; concurrent calls must not
 *    share output or workspace buffers.
 *  - Argument errors are reported synchronously, before anything is launched.
 *    Errors detected on the device (a pipeline wait that gave up) are recorded
 *    in a per-device status word read by fa_get_status().
 */
#ifndef FA_B200_H
#define FA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1, /* null/misaligned pointer, bad size, bad scale, Hq % Hkv != 0 */
  FA_ERR_UNSUPPORTED = 2, /* head dim not 64/128, device is not sm_100, size beyond limits */
  FA_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed (launch, tensor-map encode) */
  FA_ERR_TIMEOUT = 4,     /* a device-side pipeline wait gave up (see fa_get_status) */
  FA_ERR_WORKSPACE = 5    /* workspace missing or smaller than fa_bwd_workspace_size() */
} fa_status_t;

/*
 * Forward pass, padded batch (the exact tiled attention of the catalogue
 * record "Dao and colleagues: IO-aware exact attention with FlashAttention",
 * field summary).
 *   q [B,N,Hq,d], k/v [B,N,Hkv,d] bf16 (in);  o [B,N,Hq,d] bf16 (out);
 *   lse [B,Hq,N] float32 (out, natural log of the scaled scores' row sums).
 *   causal: 0 or 1 (query i sees keys 0..i).  scale: > 0 and finite, usually 1/sqrt(d).
 * B*N == 0 is a no-op returning FA_OK.
 */
fa_status_t fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                   int N, int d, int causal, float scale, void* stream);

/*
 * Forward pass, packed variable-length batch (the varlen API of the
 * Dao-AILab repository overview).
 *   q [T,Hq,d], k/v [T,Hkv,d] bf16 (in); o [T,Hq,d] bf16, lse [Hq,T] f32 (out).
 *   cu_seqlens: DEVICE int32 [nseq+1], non-decreasing, cu_seqlens[0] = 0,
 *   cu_seqlens[nseq] = total_T. max_seqlen must be >= every sequence length
 *   (rows beyond it are not computed) and <= 131072.
 * Each sequence attends only within itself; causal alignment is per sequence.
 * Output rows of empty sequences are not touched.
 */
fa_status_t fa_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                          const int* cu_seqlens, int nseq, int max_seqlen, int total_T, int Hq, int Hkv, int d,
                          int causal, float scale, void* stream);

/*
 * Forward pass with fp8-e4m3 inputs and per-block scales (contribution 3 of
 * the "FlashAttention-3: Fast and Accurate Attention with Asynchrony and
 * Low-precision" summary: FP8 GEMMs in the forward pass).
 *   q8 [B,N,Hq,d], k8/v8 [B,N,Hkv,d] e4m3 codes (in);
 *   q_scale [B,Hq,ceil(N/128)], k_scale/v_scale [B,Hkv,ceil(N/128)] float32:
 *   the value of element x of rows 128*i .. 128*i+127 of head h is code * scale[b,h,i].
 *   o [B,N,Hq,d] bf16, lse [B,Hq,N] float32 (out), as fa_fwd on the dequantised values.
 *   d must be 128.
 * S = Q K^T runs on e4m3 tensor cores (kind::f8f6f4) with the query and key
 * block scales folded into the exponent; for O += P V the e4m3 V tiles are
 * widened to f16 on chip (exactly) and P is rounded to f16 with the V block
 * scale folded in, so P keeps 11 significant bits instead of e4m3's 4.
 */
fa_status_t fa_fwd_fp8(const void* q8, const void* k8, const void* v8, const float* q_scale,
                       const float* k_scale, const float* v_scale, void* o, float* lse, int B, int Hq, int Hkv,
                       int N, int d, int causal, float scale, void* stream);

/*
 * Bytes of device workspace fa_bwd / fa_bwd_varlen need (the statistics the
 * recomputing backward of the catalogue record's summary reads back): two fp32 vectors per
 * (query head, token), the row's LSE in base 2 and D = dot(dO, O); each
 * sequence's rows start 16-byte aligned, plus 128 padding rows per head.
 * tokens = B*N (padded) or total_T (varlen); nseq = B or the number of packed
 * sequences; d does not change the size. 0 for empty inputs.
 */
size_t fa_bwd_workspace_size(int tokens, int nseq, int Hq, int d);

/*
 * Backward pass, padded batch (the catalogue record's summary: recomputation
 * instead of a stored attention matrix; the Dao-AILab repository overview:
 * deterministic backward): gradients of sum(O * dout) with respect to
 * q, k, v, recomputing the scores from q, k, v and the forward's lse.
 *   q, k, v, o, dout bf16, lse f32 (in, as produced by fa_fwd);
 *   dq [B,N,Hq,d], dk/dv [B,N,Hkv,d] bf16 (out; dk/dv summed over the query
 *   heads of each GQA group).
 *   workspace: DEVICE buffer of ws_bytes >= fa_bwd_workspace_size(B*N, B, Hq, d),
 *   256-byte aligned, contents need not be initialised (FA_ERR_WORKSPACE
 *   otherwise).
 * No atomics: every gradient element is produced by one CTA in a fixed
 * order, so results are bitwise reproducible from run to run. Three kernels
 * run on `stream`: the D/LSE preparation, dK/dV, and dQ.
 */
fa_status_t fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                   const void* dout, void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes, int B, int Hq,
                   int Hkv, int N, int d, int causal, float scale, void* stream);

/*
 * The backward pass of fa_bwd in separately launchable parts (bit mask):
 *   FA_BWD_PREPARE  D = dot(dO, O) and the base-2 LSE into the workspace;
 *   FA_BWD_DKDV     dK and dV (reads the workspace written by PREPARE);
 *   FA_BWD_DQ       dQ (reads the workspace written by PREPARE).
 * fa_bwd(...) is fa_bwd_part(FA_BWD_ALL, ...). After PREPARE has completed,
 * DKDV and DQ are independent and may run concurrently on two streams.
 * Arguments as fa_bwd; parts outside 1..7 return FA_ERR_INVALID_ARG.
 */
enum { FA_BWD_PREPARE = 1, FA_BWD_DKDV = 2, FA_BWD_DQ = 4, FA_BWD_ALL = 7 };
fa_status_t fa_bwd_part(int parts, const void* q, const void* k, const void* v, const void* o, const float* lse,
                        const void* dout, void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes, int B,
                        int Hq, int Hkv, int N, int d, int causal, float scale, void* stream);

/*
 * Backward pass without any device allocation, for callers that cannot
 * allocate device memory themselves: runtimes that plan all device memory
 * ahead of time and forbid further allocations while they run, plugins that
 * have no access to their host's allocator, and code whose memory budget is
 * fixed once at start-up. (No counterpart in the pages: this is a library
 * convenience.)
 *   Arguments and results as fa_bwd, minus the workspace: the scratch lives in
 *   an 8 MiB array inside the library, on every device that loads it, for the
 *   life of the process. It runs exactly what fa_bwd runs (bitwise the same
 *   results). The problem must fit the array:
 *   fa_bwd_workspace_size(B*N, B, Hq, d) <= 8 MiB,
 *   i.e. Hq * (B*N + 4*B + 131) up to about 1.04 million; larger problems
 *   return FA_ERR_WORKSPACE and launch nothing.
 *   Set-up on the first call on each device, with that device current: the
 *   array's device address is looked up (cudaGetSymbolAddress), and, as for
 *   the first fa_bwd on a device, a second stream and two events are created
 *   (the dQ kernel runs on that stream beside the dK/dV kernel). Make that
 *   first call before any stream capture.
 *   Every call uses the same array: calls whose work overlaps on the GPU (on
 *   different streams, or from different threads) race on it and must be
 *   serialised by the caller. The array keeps whatever the last call left;
 *   nothing in it needs clearing between calls.
 *   No cudaMalloc, cudaFree or other allocating routine is called.
 *   The library caches per-device state (these addresses, the stream and the
 *   events) for the life of the process: cudaDeviceReset while it is loaded
 *   is not supported.
 */
fa_status_t fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                           const void* dout, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N, int d,
                           int causal, float scale, void* stream);

/* Backward pass, packed variable-length batch (the varlen API of the
 * Dao-AILab repository overview; recomputation as fa_bwd); layouts as
 * fa_fwd_varlen. */
fa_status_t fa_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const float* lse,
                          const void* dout, void* dq, void* dk, void* dv, void* workspace, size_t ws_bytes,
                          const int* cu_seqlens, int nseq, int max_seqlen, int total_T, int Hq, int Hkv, int d,
                          int causal, float scale, void* stream);

/*
 * Decode: Nq new query rows per sequence against a key/value cache (the
 * KV-cache API of the Dao-AILab repository overview), split over the cache
 * and combined through the per-split log-sum-exp.
 *   q [B,Nq,Hq,d] bf16; k_cache/v_cache [B,Ncache,Hkv,d] bf16 (in);
 *   cache_seqlens: DEVICE int32 [B], valid cache rows L_b per sequence
 *   (clamped to 0..Ncache); o [B,Nq,Hq,d] bf16, lse [B,Hq,Nq] f32 (out).
 *   Query i is position L_b - Nq + i of its sequence: with causal = 1 it sees
 *   keys 0 .. L_b - Nq + i, otherwise keys 0 .. L_b - 1. A row that sees no
 *   key gets O = 0 and LSE = -inf.
 *   Nq * (Hq/Hkv) <= 16 (FA_ERR_UNSUPPORTED otherwise); d = 64 or 128.
 *   num_splits >= 1: the cache is cut into that many ranges of whole 128-key
 *   tiles (fewer if Ncache is short); with more than one range the partial
 *   results go to `workspace` (DEVICE, 16-byte aligned, at least
 *   fa_fwd_kvcache_workspace_size(B, Nq, Hq, d, num_splits) bytes) and a second
 *   kernel merges them. Bound by HBM bandwidth: the cache is read once.
 */
fa_status_t fa_fwd_kvcache(const void* q, const void* k_cache, const void* v_cache, const int* cache_seqlens,
                           void* o, float* lse, void* workspace, size_t ws_bytes, int B, int Nq, int Hq, int Hkv,
                           int Ncache, int d, int causal, float scale, int num_splits, void* stream);

/* Workspace bytes of fa_fwd_kvcache (0 when num_splits <= 1). */
size_t fa_fwd_kvcache_workspace_size(int B, int Nq, int Hq, int d, int num_splits);

/*
 * Split count fa_fwd_kvcache runs fastest with on the current device for B
 * sequences, Hkv key/value heads, a cache of Ncache rows and head dim d: one
 * persistent CTA per SM streams (sequence, kv head, split) units back to back;
 * the count trades idle SMs against per-unit and merge costs (a launch-time
 * model with constants measured on B200). Returns 1 for invalid sizes or when
 * no CUDA device is usable. Not in the pages (a host-side choice).
 */
int fa_fwd_kvcache_num_splits(int B, int Hkv, int Ncache, int d);

/*
 * Forward pass with a block-sparse mask (the topic page's block-sparse
 * variant, which it calls approximate: only the listed blocks are attended;
 * the mask layout is a reading). As fa_fwd, plus
 *   block_mask DEVICE uint8 [Hq][nb][nb], nb = ceil(N/128): key block j
 *              (keys 128j .. 128j+127) is visible to query block i of query
 *              head h when block_mask[h][i][j] != 0; the same mask for every
 *              sequence of the batch; with causal = 1 the causal mask applies
 *              too.
 * Only visited key blocks are loaded and multiplied. A query row that sees no
 * key gets O = 0 and LSE = -inf. NULL mask: FA_ERR_INVALID_ARG; N > 131072:
 * FA_ERR_UNSUPPORTED.
 */
fa_status_t fa_fwd_blocksparse(const void* q, const void* k, const void* v, const unsigned char* block_mask, void* o,
                               float* lse, int B, int Hq, int Hkv, int N, int d, int causal, float scale,
                               void* stream);

/*
 * Backward pass of fa_fwd_blocksparse: the gradient of the same block-masked
 * attention (the backward of the topic page's backward-pass section with P
 * recomputed only on visible blocks; entries of hidden blocks are exactly 0,
 * so they add nothing to dQ, dK or dV). Arguments as fa_bwd, plus block_mask
 * exactly as given to fa_fwd_blocksparse (DEVICE uint8 [Hq][nb][nb]); o and
 * lse are that call's outputs (a row with lse = -inf gets dQ = 0). dQ units
 * visit only the key blocks their query tile sees; dK/dV units only the
 * (query head, query tile) steps that see their key tile, following a work
 * plan made on the device: a unit more than twice the average unit long (a
 * key block every query block sees) is split into chunks of about the
 * average, whose fp32 partial sums are added in chunk order afterwards. A
 * tile that sees nothing writes zeros. Deterministic.
 *   workspace: ws_bytes >= fa_bwd_blocksparse_workspace_size(B, Hq, Hkv, N, d)
 *   (the two vectors of fa_bwd plus the plan and four partial [128][d] fp32
 *   pairs per SM of the current device), 256-byte aligned; FA_ERR_WORKSPACE
 *   otherwise. NULL mask: FA_ERR_INVALID_ARG.
 */
fa_status_t fa_bwd_blocksparse(const void* q, const void* k, const void* v, const unsigned char* block_mask,
                               const void* o, const float* lse, const void* dout, void* dq, void* dk, void* dv,
                               void* workspace, size_t ws_bytes, int B, int Hq, int Hkv, int N, int d, int causal,
                               float scale, void* stream);

/* Workspace bytes fa_bwd_blocksparse needs on the current device; 0 for
 * invalid sizes or when no device is available. */
size_t fa_bwd_blocksparse_workspace_size(int B, int Hq, int Hkv, int N, int d);

/*
 * Block-scaled e4m3 inputs for fa_fwd_fp8, with optional incoherent
 * processing (the FA-3 summary's lower-error FP8, contribution 3; the
 * technique is not named there, this rotation is the reading taken): with
 * rotate = 1 each row is first multiplied by the orthogonal Hadamard matrix
 * H_d / sqrt(d) (Sylvester's construction; fast Walsh-Hadamard butterflies in
 * fp32, stage widths 1, 2, ..., d/2, then one multiply by fp32(1/sqrt(d))).
 * Rotate Q and K, not V: (Q H)(K H)^T = Q K^T.
 *   x      DEVICE bf16 [B,N,H,d], 8-byte aligned (in);
 *   codes  DEVICE e4m3 [B,N,H,d], 4-byte aligned (out);
 *   scales DEVICE fp32 [B,H,ceil(N/128)] (out): per (batch, head, 128-row
 *          block) s = amax / 448 in fp32 (1 for an all-zero block); codes are
 *          the round-to-nearest-even e4m3 of the fp32 quotient (x or x H/sqrt d) / s.
 *   d = 64 or 128. One kernel on `stream`, bound by HBM.
 */
fa_status_t fa_fp8_quantize(const void* x, void* codes, float* scales, int B, int N, int H, int d, int rotate,
                            void* stream);

/*
 * The inverse of fa_fp8_quantize, input of the fp8 backward: bf16 values in
 * the original space from block-scaled e4m3 codes. The fp8 forward attends
 * over code * scale (Q, K rotated when quantised with rotate = 1); its
 * gradient (straight-through reading: the pages describe an fp8 forward
 * only) is the bf16 backward (fa_bwd, with the fp8 forward's O and LSE) on
 * these values, with the rotation undone for Q and K, which keeps Q K^T.
 *   codes  DEVICE e4m3 [B,N,H,d], 4-byte aligned (in);
 *   scales DEVICE fp32 [B,H,ceil(N/128)] (in), as fa_fp8_quantize writes them;
 *   x      DEVICE bf16 [B,N,H,d], 8-byte aligned (out): per element, in fp32,
 *          code * scale; with unrotate = 1 then the butterflies of the fast
 *          Walsh-Hadamard transform and a multiply by fp32(1/sqrt(d))
 *          (H_d / sqrt(d) is its own inverse); rounded to nearest even bf16.
 *   d = 64 or 128. One kernel on `stream`, bound by HBM.
 */
fa_status_t fa_fp8_dequantize(const void* codes, const float* scales, void* x, int B, int N, int H, int d,
                              int unrotate, void* stream);

/*
 * The fp8 backward with its score products on the e4m3 codes (FA-3 summary,
 * contribution 3: FP8 GEMMs), for the output of fa_fwd_fp8: as fa_bwd, except
 * that S = Q K^T (dQ kernel) and S^T = K Q^T (dK/dV kernel) run on the codes
 * (tcgen05 kind::f8f6f4, fp32 sums) with the block scales folded into the
 * exponent, exactly as fa_fwd_fp8 forms its scores, so P matches the forward's
 * LSE. The other products (dV = P^T dO, dK = dS^T Q, dQ = dS K, dP = dO V^T)
 * stay 16-bit: P and dS rounded to e4m3 would leave about 2.5% RMS error in
 * the gradients, past their 1e-2 bound.
 *   q8, k8   DEVICE e4m3 codes [B,N,Hq,128], [B,N,Hkv,128], 16-byte aligned,
 *            as given to fa_fwd_fp8 (rotated or not; S is the same either way);
 *   q_scale, k_scale DEVICE fp32 [B,H,ceil(N/128)] block scales of those codes;
 *   q, k, v  DEVICE bf16 values of the other products, in the original space:
 *            fa_fp8_dequantize of the codes (Q and K with `unrotate` when the
 *            codes were rotated);
 *   o, lse   fa_fwd_fp8's output on these codes; dout, dq, dk, dv, workspace,
 *            ws_bytes and the rest as fa_bwd (workspace fa_bwd_workspace_size).
 *   d = 128 only (FA_ERR_UNSUPPORTED otherwise); null or misaligned code or
 *   scale pointers return FA_ERR_INVALID_ARG. Deterministic; launches as fa_bwd.
 */
fa_status_t fa_bwd_fp8(const void* q8, const void* k8, const float* q_scale, const float* k_scale, const void* q,
                       const void* k, const void* v, const void* o, const float* lse, const void* dout, void* dq,
                       void* dk, void* dv, void* workspace, size_t ws_bytes, int B, int Hq, int Hkv, int N, int d,
                       int causal, float scale, void* stream);

/*
 * Merge of attention partials over disjoint key sets (the multi-GPU variants
 * of the topic page "Flash Attention and Efficient Transformer Mechanisms";
 * used by context-parallel ring attention): partial t is exact attention of
 * the same query rows over key shard t, normalised by its own softmax sum, as
 * fa_fwd writes it; over all shards
 *   lse = log sum_t exp lse_t,   o = sum_t exp(lse_t - lse) o_t.
 *   o_parts   DEVICE bf16 [nparts][B,N,H,d], 16-byte aligned (in);
 *   lse_parts DEVICE fp32 [nparts][B,H,N] natural log (in; -inf for a row of a
 *             partial that saw no key);
 *   o DEVICE bf16 [B,N,H,d], 16-byte aligned; lse DEVICE fp32 [B,H,N] (out).
 *   nparts >= 1; d = 64 or 128. The sums run in fp32. One HBM-bound kernel
 *   on `stream`.
 */
fa_status_t fa_attn_merge(const void* o_parts, const float* lse_parts, int nparts, void* o, float* lse, int B, int N,
                          int H, int d, void* stream);


/*
 * Sum of gradient partials over key blocks (context-parallel ring attention
 * backward: the dQ, dK, dV contributions of the key shards):
 *   acc[i] = (first ? 0 : acc[i]) + part[i];  out[i] = bf16(acc[i]) if out.
 *   acc  DEVICE fp32 [count], 16-byte aligned (in/out);
 *   part DEVICE bf16 [count], 16-byte aligned, or NULL (adds nothing);
 *   out  DEVICE bf16 [count], 16-byte aligned, or NULL.
 *   count a multiple of 8. One elementwise kernel on `stream`.
 * The pages have no counterpart; it is the sum in the gradient of a
 * partitioned key set.
 */
fa_status_t fa_grad_accumulate(float* acc, const void* part, void* out, long long count, int first, void* stream);

/*
 * Synchronises `stream`, then returns and clears the device-side status word
 * of the current device (FA_OK if no kernel reported an error since the last
 * call). Returns FA_ERR_CUDA if the synchronisation itself failed.
 */
fa_status_t fa_get_status(void* stream);

/* Raw device status word of the last fa_get_status() that found an error
 * (low byte: status code; bits 8..15: id of the wait that gave up). */
int fa_last_device_error_word(void);

/* Human-readable name of a status code (static storage). */
const char* fa_status_string(fa_status_t status);

/*
 * Upper bound, in nanoseconds, of every device-side pipeline wait of kernels
 * launched after this call (default 4e9). A wait that runs out records
 * FA_ERR_TIMEOUT and the kernel exits cleanly instead of hanging.
 */
void fa_set_wait_timeout_ns(uint64_t ns);

/*
 * Test hook: when set to 1, the next forward launches never load their first
 * K tile, so the pipeline waits run out and FA_ERR_TIMEOUT is recorded (used
 * to test the bounded-wait path without faulting the GPU). 0 restores normal
 * operation.
 */
void fa_debug_set_inject(int mode);


#ifdef __cplusplus
}
#endif

#endif /* FA_B200_H */
