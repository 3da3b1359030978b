/*
 * attn.h -- C ABI of the B200 (sm_100a) fused attention library
 * (libattn_sm100.so).
 *
 * Operations, all on one GPU:
 *
 *   attn_fwd / attn_fwd_fp8 / attn_fwd_e5m2 / attn_fwd_mla
 *                             fused, tiled scaled-dot-product attention
 *                             O = softmax(scale * Q K^T + mask) V, with the
 *                             per-row log-sum-exp, computed with the online
 *                             softmax recurrence (running row max and sum,
 *                             accumulator rescaled at each K/V block) so the
 *                             score matrix never reaches HBM.
 *   attn_decode_paged         one query token per sequence against a KV cache
 *                             held in fixed-size pages addressed through a
 *                             block table, split over the cache and merged by
 *                             log-sum-exp (attn_decode_paged_multi: the last
 *                             q_len cached tokens; attn_decode_paged_mla: keys
 *                             and values of different widths;
 *                             attn_decode_paged_noalloc: scratch inside the
 *                             library).
 *   attn_prefill_paged        a chunk of new tokens against the paged cache
 *                             (chunked prefill), with attn_kv_append writing
 *                             the chunk's K/V into its pages.
 *   attn_bwd                  gradients dQ, dK, dV of attn_fwd, recomputing
 *                             the weights from the forward's LSE.
 *
 * Sources (page title, section):
 *   - "003-注意力机制详解：从基础Attention到DeepSeek的优化策略" (lakecityint.com),
 *     §一 attention_naive / safe_softmax (the definition), §二 the tiled
 *     FlashAttention loop (online softmax), §三.1 mixed precision (fp16/bf16
 *     operands, fp32 softmax and accumulation), §三.2 sliding window.
 *   - "LLM 中的 Attention 实现及优化" (zeeklog.com): MQA/GQA with repeat_kv and
 *     the (batch, heads, seqlen, head_dim) layout; the KV-cache size formula;
 *     sliding-window attention; PagedAttention.
 *   - MQA / GQA / Flash Attention article (tqpw.cn) §2.1 (MQA), §3.1 (GQA,
 *     h % g == 0), §4.1-4.2 (tiling into SRAM, online softmax, one fused
 *     kernel).
 *   - "注意力机制深度优化" (kler.cn) §一.1 (FP8 e4m3), §一.2 (skipping the
 *     upper-right causal triangle), §四.2 (FP8 e5m2).
 *   - "高效多头潜在注意力解码技术：Flash MLA深度解析" (developer.baidu.com)
 *     §2.1: queries and keys in a latent dimension, values in their own.
 *
 * Conventions shared by every entry point
 *   - Pointers are DEVICE pointers unless stated otherwise.  The caller owns
 *     every buffer (inputs, outputs and the decode workspace); the library
 *     allocates no device memory on any call.  Its only device state is one
 *     status word per GPU, created when the library is loaded.
 *   - All launches are asynchronous on the caller's CUDA stream `stream`
 *     (a cudaStream_t passed as void*; NULL = legacy default stream).
 *     The decode kernels are launched as programmatic dependents of the
 *     kernel before them in the stream: they may become resident, set up and
 *     read seq_lens and block_table early, while that kernel still runs;
 *     queries, pages, the workspace and the outputs are read or written only
 *     after it has completed.  So the kernel immediately before a decode call
 *     (attn_decode_paged*) in the same stream must not write that call's
 *     seq_lens or block_table; with any other operation between them (a copy,
 *     an event, another kernel) stream order holds as for a plain launch.
 *   - A call returns ATTN_OK once its kernels are enqueued.  Argument errors
 *     are detected on the host before anything is launched and return
 *     ATTN_ERR_INVALID / ATTN_ERR_UNSUPPORTED with nothing written.  A CUDA
 *     launch failure returns ATTN_ERR_CUDA.  Errors found by the kernels
 *     themselves (a bounded wait that ran out, an out-of-range page id in
 *     bounds-check mode) are recorded in the device status word and reported
 *     by attn_last_device_error().  The kernels never trap.
 *   - Tensors are contiguous, row-major, with a 16-byte aligned base.
 *   - Per-device state (the status word's address, kernel attributes) is
 *     looked up on first use on each device and cached for the life of the
 *     process; after cudaDeviceReset the library must not be used again in
 *     that process.
 */
#ifndef ATTN_SM100_H
#define ATTN_SM100_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
#define ATTN_API extern "C" __attribute__((visibility("default")))
#else
#define ATTN_API __attribute__((visibility("default")))
#endif

typedef void* attn_stream_t; /* cudaStream_t of the caller */

enum attn_status {
  ATTN_OK = 0,
  ATTN_ERR_INVALID = -1,     /* bad argument (shape, pointer, alignment) */
  ATTN_ERR_UNSUPPORTED = -2, /* valid but not built (e.g. head_dim 96)   */
  ATTN_ERR_CUDA = -3,        /* a CUDA runtime/driver call failed         */
  ATTN_ERR_TIMEOUT = -4,     /* a kernel's bounded wait ran out           */
  ATTN_ERR_BOUNDS = -5       /* bounds-check mode found a bad index       */
};

/*
 * attn_fwd -- bf16 fused attention forward (prefill).
 *
 *   q    [B, Hq,  Lq, D] bf16     k, v [B, Hkv, Lk, D] bf16
 *   o    [B, Hq,  Lq, D] bf16 (written)
 *   lse  [B, Hq,  Lq]    fp32 (written; may be NULL): natural-log
 *        log-sum-exp of the scaled, masked logits of each row.
 *
 * Layout (batch, heads, seqlen, head_dim) as produced by
 * view(...).transpose(1, 2) in the zeeklog page's GQA code.  Query head h reads
 * K/V head h / (Hq / Hkv): MHA (Hkv == Hq), GQA (Hq % Hkv == 0) and MQA
 * (Hkv == 1).  Scores are scale * q.k accumulated in fp32; softmax in fp32; P
 * is rounded to bf16 for the P.V product; O is accumulated in fp32 and rounded
 * to bf16 once (mixed-precision scheme of the lakecityint.com page §三.1).
 *
 * Masks:
 *   causal = 0: every query sees all Lk keys.
 *   causal = 1: query i sees keys 0 .. i + (Lk - Lq) (the triangle is aligned
 *     to the bottom-right corner; with Lq == Lk this is keys 0..i).  K/V blocks
 *     entirely above the diagonal are never loaded or multiplied.
 *   window W > 0 (requires causal = 1): query i sees the W keys
 *     max(0, i' - W + 1) .. i' with i' = i + (Lk - Lq).  Blocks entirely before
 *     the window are never loaded.  window <= 0: no window.
 * A row that sees no key (only possible when Lq > Lk with causal = 1, or
 * Lk == 0) gets O = 0 and LSE = -inf.
 *
 * Supported: D in {64, 128}; 1 <= Hkv <= Hq, Hq % Hkv == 0; B, Lq >= 0;
 * Lk >= 0; any Lq, Lk (ragged tails are handled).  Returns ATTN_ERR_INVALID
 * for bad shapes, NULL or misaligned pointers, window > 0 without causal;
 * ATTN_ERR_UNSUPPORTED for other D.
 */
ATTN_API int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                      int B, int Hq, int Hkv, int Lq, int Lk, int D,
                      float scale, int causal, int window, attn_stream_t stream);

/*
 * attn_fwd_fp8 -- the same operation on float8_e4m3fn inputs (the e4m3 FP8
 * format of the kler.cn page §一.1), bf16 output.
 *
 *   q, k, v  e4m3 bytes, same shapes/layout as attn_fwd; o bf16; lse fp32.
 *   q_descale, k_descale, v_descale: per-tensor scales, i.e. the real value of
 *   an element is e4m3_value * descale.  The logits are
 *   scale * q_descale * k_descale * (q8 . k8); P is quantised to e4m3 for the
 *   P.V product (values in [0, 256]); O is multiplied by v_descale.
 *
 * Supported: D == 128 only (ATTN_ERR_UNSUPPORTED otherwise).
 */
ATTN_API int attn_fwd_fp8(const void* q, const void* k, const void* v, void* o, float* lse,
                          int B, int Hq, int Hkv, int Lq, int Lk, int D,
                          float scale, int causal, int window,
                          float q_descale, float k_descale, float v_descale,
                          attn_stream_t stream);

/*
 * attn_fwd_e5m2 -- attn_fwd_fp8 on float8_e5m2 inputs (the e5m2 FP8 format of
 * the kler.cn page §四.2, "torch_dtype=torch.float8_e5m2"), bf16 output.
 *
 *   q, k, v  e5m2 bytes, same shapes/layout as attn_fwd; o bf16; lse fp32.
 *   q_descale, k_descale, v_descale: per-tensor scales as attn_fwd_fp8.
 * The logits come from an e5m2 x e5m2 product with fp32 accumulation.  The
 * weights P (fp32 softmax, scaled by 2^8 with an exact running max) are
 * multiplied with V in e5m2 -- one operand type per product -- as two terms,
 * e5m2(P) and the e5m2 rounding residual of P, so each weight carries about 6
 * significant bits (e5m2 alone has 3); O is multiplied by v_descale.
 *
 * Supported: D == 128 only (ATTN_ERR_UNSUPPORTED otherwise).
 */
ATTN_API int attn_fwd_e5m2(const void* q, const void* k, const void* v, void* o, float* lse,
                           int B, int Hq, int Hkv, int Lq, int Lk, int D,
                           float scale, int causal, int window,
                           float q_descale, float k_descale, float v_descale,
                           attn_stream_t stream);

/*
 * attn_fwd_mla -- bf16 attention forward whose queries and keys have another
 * width than the values, up to 256: attention in a latent space, where q and
 * k are projections to a latent dimension (64-256 on the page) and v to its
 * own value dimension (latent projection of the page "高效多头潜在注意力解码
 * 技术：Flash MLA深度解析", §2.1).
 *
 *   q    [B, Hq,  Lq, D_qk] bf16     k [B, Hkv, Lk, D_qk] bf16
 *   v    [B, Hkv, Lk, D_v]  bf16
 *   o    [B, Hq,  Lq, D_v]  bf16 (written)
 *   lse  [B, Hq,  Lq]       fp32 (written; may be NULL)
 *
 * Masks, GQA/MQA head mapping, scale, precision and empty-row behaviour as
 * attn_fwd.  One 128-row query tile per SM with 64-key K/V blocks (two
 * 128-row accumulators of 256 columns do not fit the tensor memory), so for
 * D_qk = D_v in {64, 128} attn_fwd is the faster call.
 * Supported: D_qk, D_v in {64, 128, 192, 256} (ATTN_ERR_UNSUPPORTED
 * otherwise); other checks as attn_fwd.
 */
ATTN_API int attn_fwd_mla(const void* q, const void* k, const void* v, void* o, float* lse,
                          int B, int Hq, int Hkv, int Lq, int Lk, int D_qk, int D_v,
                          float scale, int causal, int window, attn_stream_t stream);

/*
 * attn_bwd_workspace_bytes -- scratch attn_bwd needs: an fp32 dQ accumulator
 * of B * Hq * Lq * D floats plus two floats per query row (LSE in log2 units
 * and rowsum(dO * O)): B * Hq * Lq * (D + 2) * 4 bytes.  0 for empty shapes.
 */
ATTN_API size_t attn_bwd_workspace_bytes(int B, int Hq, int Lq, int D);

/*
 * attn_bwd -- gradients of attn_fwd (no counterpart call in the pages, which
 * describe the backward only as recomputing the attention weights from
 * stored statistics instead of keeping them: tqpw.cn article §4.1).
 *
 *   q, k, v, o   as attn_fwd (o = its output), bf16
 *   dout         [B, Hq, Lq, D] bf16: gradient of the loss with respect to O
 *   lse          [B, Hq, Lq] fp32: attn_fwd's LSE (natural log)
 *   dq           [B, Hq, Lq, D] bf16 (written)
 *   dk, dv       [B, Hkv, Lk, D] bf16 (written; each K/V head sums its group)
 *   workspace    at least attn_bwd_workspace_bytes(B, Hq, Lq, D) bytes;
 *                contents on entry do not matter
 *   scale, causal, window as attn_fwd (same mask, same alignment); a row
 *                that sees no key (causal with Lq > Lk) gets dQ = 0 and adds
 *                nothing to dK, dV
 *
 * P = exp(scale * q k^T - lse) is recomputed, rounded to bf16 for the
 * dV = P^T dO product, and dS = P * (dP - rowsum(dO * O)) to bf16 for the
 * dK and dQ products; accumulation in fp32.  Supported: bf16, D in {64, 128}.
 * dK and dV are the same bits on every call.  dQ sums one fp32 partial per
 * 128-key tile in whatever order the tiles finish, so it can differ between
 * calls in the last bits of its fp32 sum (before its rounding to bf16).
 */
ATTN_API int attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                      const float* lse, void* dq, void* dk, void* dv,
                      int B, int Hq, int Hkv, int Lq, int Lk, int D,
                      float scale, int causal, int window,
                      void* workspace, size_t workspace_bytes, attn_stream_t stream);

/*
 * attn_decode_workspace_bytes -- size of the scratch buffer attn_decode_paged
 * needs for these sizes: per query head of every sequence, up to
 * S = ceil(max_pages_per_seq / 32) + 1 partial results of D + 1 floats
 * (B * Hq * S * (D + 1) * 4 bytes; D is the value width).  Host only; never
 * fails (0 for empty shapes).
 */
ATTN_API size_t attn_decode_workspace_bytes(int B, int Hq, int max_pages_per_seq, int D);

/*
 * attn_decode_paged -- single-token decode against a paged KV cache
 * (PagedAttention section of the zeeklog page: non-contiguous small-block KV
 * storage), split over the cache and merged by log-sum-exp.
 *
 *   q           [B, Hq, D] bf16, one query token per sequence
 *   k_pages     [num_pages, page_size, Hkv, D] bf16, shared pool
 *   v_pages     [num_pages, page_size, Hkv, D] bf16
 *   block_table [B, max_pages_per_seq] int32: page id of each page of each
 *               sequence (entries past a sequence's length are not read)
 *   seq_lens    [B] int32 (device), 0 <= seq_lens[b] <= max_pages_per_seq *
 *               page_size (longer lengths are clamped to that)
 *   o           [B, Hq, D] bf16 (written)
 *   lse         [B, Hq] fp32 (written; may be NULL)
 *   workspace   caller-owned device scratch of at least
 *               attn_decode_workspace_bytes(B, Hq, max_pages_per_seq, D) bytes;
 *               its contents on entry do not matter, but two calls that may
 *               run at the same time must not share one.
 *
 * The single query sees every cached key (causal alignment at the
 * bottom-right corner); cache slots past seq_lens[b] in a sequence's last
 * page are never used, whatever they hold.  seq_lens[b] == 0 gives O = 0 and
 * LSE = -inf.
 * Supported: page_size == 16, D in {64, 128, 192, 256}, Hq % Hkv == 0 and
 * Hq / Hkv <= 128 (otherwise ATTN_ERR_UNSUPPORTED).
 * Page ids are trusted unless bounds-check mode is on (attn_set_debug), in
 * which case an id outside [0, num_pages) reads as a page of zeros and is
 * reported as ATTN_ERR_BOUNDS by attn_last_device_error().  Pages are copied
 * by the tensor-memory-access unit against the pool's bounds, so an untrusted
 * id cannot make the kernel read outside the pool either way.
 */
ATTN_API int attn_decode_paged(const void* q, const void* k_pages, const void* v_pages,
                               const int* block_table, const int* seq_lens, void* o, float* lse,
                               int B, int Hq, int Hkv, int D, int page_size, int num_pages,
                               int max_pages_per_seq, float scale,
                               void* workspace, size_t workspace_bytes, attn_stream_t stream);

/*
 * attn_decode_paged_multi -- attn_decode_paged for q_len new tokens per
 * sequence (speculative-decoding verification, chunked decode): the last
 * q_len cached tokens of each sequence are the queries, and query token i
 * (0-based) sees the cached tokens 0 .. seq_lens[b] - q_len + i (the causal
 * mask aligned at the bottom-right corner, as in attn_fwd).  Their K/V must
 * already be in the cache.  (Not a call the pages define: the same
 * PagedAttention decode with a causal block of queries.)
 *
 *   q      [B, Hq, q_len, D] bf16
 *   o      [B, Hq, q_len, D] bf16 (written)
 *   lse    [B, Hq, q_len] fp32 (written; may be NULL)
 *   workspace  at least attn_decode_workspace_bytes(B, Hq * q_len,
 *              max_pages_per_seq, D) bytes
 *   everything else as attn_decode_paged.
 *
 * A query token with no cached token at or before its position (seq_lens[b]
 * < q_len) gets O = 0 and LSE = -inf.
 * Supported: as attn_decode_paged, with (Hq / Hkv) * q_len <= 128 (otherwise
 * ATTN_ERR_UNSUPPORTED); q_len >= 1 (q_len = 1 is attn_decode_paged).
 */
ATTN_API int attn_decode_paged_multi(const void* q, const void* k_pages, const void* v_pages,
                                     const int* block_table, const int* seq_lens, void* o, float* lse,
                                     int B, int Hq, int Hkv, int q_len, int D, int page_size, int num_pages,
                                     int max_pages_per_seq, float scale,
                                     void* workspace, size_t workspace_bytes, attn_stream_t stream);

/*
 * attn_decode_paged_mla -- attn_decode_paged_multi with keys and values of
 * different widths: queries and keys of width D_qk, values of width D_v,
 * attention in a latent space (latent projection of the page "高效多头潜在
 * 注意力解码技术：Flash MLA深度解析", §2.1) against a paged cache.
 *
 *   q        [B, Hq, q_len, D_qk] bf16: the last q_len cached tokens
 *   k_pages  [num_pages, page_size, Hkv, D_qk] bf16
 *   v_pages  [num_pages, page_size, Hkv, D_v] bf16 (same page ids as k_pages)
 *   o        [B, Hq, q_len, D_v] bf16 (written); lse [B, Hq, q_len] fp32
 *            (written; may be NULL)
 *   workspace  at least attn_decode_workspace_bytes(B, Hq * q_len,
 *              max_pages_per_seq, D_v) bytes
 *   everything else as attn_decode_paged_multi.
 *
 * Supported: D_qk, D_v in {64, 128, 192, 256}, page_size == 16,
 * (Hq / Hkv) * q_len <= 128 (otherwise ATTN_ERR_UNSUPPORTED).  With
 * D_v > 128 the tensor memory holds one decode CTA per SM instead of two.
 */
ATTN_API int attn_decode_paged_mla(const void* q, const void* k_pages, const void* v_pages,
                                   const int* block_table, const int* seq_lens, void* o, float* lse,
                                   int B, int Hq, int Hkv, int q_len, int D_qk, int D_v,
                                   int page_size, int num_pages, int max_pages_per_seq, float scale,
                                   void* workspace, size_t workspace_bytes, attn_stream_t stream);

/*
 * attn_prefill_paged -- chunked prefill over a paged KV cache: the last Lq
 * cached tokens of every sequence are the queries, and query token i sees the
 * cached tokens 0 .. seq_lens[b] - Lq + i (the causal mask aligned at the
 * bottom-right corner, as in attn_fwd; with window > 0 only the last window
 * of them).  Their K/V must already be in the pool (attn_kv_append).  The
 * same tiled kernel as attn_fwd, its K/V tiles gathered page by page through
 * the block table (PagedAttention section of the zeeklog page).
 *
 *   q           [B, Hq, Lq, D] bf16
 *   k_pages     [num_pages, page_size, Hkv, D] bf16, shared pool (num_pages >= 1)
 *   v_pages     [num_pages, page_size, Hkv, D] bf16
 *   block_table [B, max_pages_per_seq] int32 (entries past a sequence's length
 *               are not read)
 *   seq_lens    [B] int32 (device): cached tokens, the Lq new ones included;
 *               clamped to max_pages_per_seq * page_size
 *   o           [B, Hq, Lq, D] bf16 (written); lse [B, Hq, Lq] fp32 (written;
 *               may be NULL)
 *
 * Rows without any visible token get O = 0, LSE = -inf; cache slots past
 * seq_lens[b] are never used, whatever they hold.  Page ids are read through
 * the pool's tensor map: an id outside the pool reads zeros, never faults.
 * Supported: bf16, D in {64, 128}, page_size == 16, Hq % Hkv == 0.
 */
ATTN_API int attn_prefill_paged(const void* q, const void* k_pages, const void* v_pages,
                                const int* block_table, const int* seq_lens, void* o, float* lse,
                                int B, int Hq, int Hkv, int Lq, int D, int page_size, int num_pages,
                                int max_pages_per_seq, float scale, int window, attn_stream_t stream);

/*
 * attn_kv_append -- write the K/V of each sequence's L_new newest tokens into
 * their slots of the page pools: token t of sequence b goes to position
 * seq_lens[b] - L_new + t (seq_lens counts the new tokens), i.e. page
 * block_table[b][pos / page_size], slot pos % page_size.  Positions below 0
 * are skipped.
 *
 *   k_new, v_new  [B, Hkv, L_new, D] bf16 (read)
 *   k_pages, v_pages, block_table, seq_lens as attn_prefill_paged (pools written)
 *
 * Every page id is checked before the write: one outside [0, num_pages) is
 * skipped and reported as ATTN_ERR_BOUNDS by attn_last_device_error().
 * Supported: D a multiple of 8, page_size == 16.
 */
ATTN_API int attn_kv_append(const void* k_new, const void* v_new, void* k_pages, void* v_pages,
                            const int* block_table, const int* seq_lens, int B, int Hkv, int L_new, int D,
                            int page_size, int num_pages, int max_pages_per_seq, attn_stream_t stream);

/*
 * attn_decode_paged_noalloc -- attn_decode_paged for callers that cannot
 * allocate device memory at the call site (no counterpart in the pages this
 * library follows).
 *
 * Who needs it: code running inside another runtime's execution hook (an
 * engine plugin's enqueue, for instance) where that runtime owns all device
 * memory and no allocation is allowed, or a service that must not grow its
 * device footprint after start-up; a cudaMalloc there would also synchronise
 * the device.  Here the decode scratch is a fixed device array compiled into
 * the library (ATTN_DECODE_NOALLOC_SCRATCH_BYTES, held by every GPU that loads
 * the library until the process exits), so the call allocates nothing:
 * no cudaMalloc, cudaFree or allocating library routine.
 *
 * Arguments, layouts, supported sizes, argument checks and results are those
 * of attn_decode_paged, without the workspace.  Sizes that pass those checks
 * but whose scratch (attn_decode_workspace_bytes) exceeds the array return
 * ATTN_ERR_INVALID before anything is launched, with the sizes in
 * attn_last_error_message().
 * Set-up: the CUDA runtime loads the array onto a GPU when it is first needed
 * there -- under lazy module loading (the default), at the first call of this
 * entry point on that device, which looks up the array's address.  That first
 * call per device therefore allocates the array and may synchronise: make it
 * once at start-up, with the device current, outside any context that forbids
 * allocation or synchronisation and before any stream capture (a call with
 * B == 0 does only this set-up).  Later calls on that device allocate nothing.
 * All calls share the one array and it keeps the previous call's contents
 * (nothing in it needs to start at zero); calls that overlap on the GPU --
 * different streams with no ordering between them -- race on it.  The array's
 * address is cached per device for the process: after cudaDeviceReset this
 * library (which caches its other per-device state the same way) must not be
 * used again in that process.
 */
#define ATTN_DECODE_NOALLOC_SCRATCH_BYTES (32u << 20)
ATTN_API int attn_decode_paged_noalloc(const void* q, const void* k_pages, const void* v_pages,
                                       const int* block_table, const int* seq_lens, void* o, float* lse,
                                       int B, int Hq, int Hkv, int D, int page_size, int num_pages,
                                       int max_pages_per_seq, float scale, attn_stream_t stream);

/*
 * attn_last_device_error -- synchronises `stream`, then returns and clears the
 * status word the kernels write on the current device: ATTN_OK,
 * ATTN_ERR_TIMEOUT (a bounded wait inside a kernel ran out; the kernel
 * released its resources and returned), ATTN_ERR_BOUNDS, or ATTN_ERR_CUDA if
 * the synchronisation itself failed.
 */
ATTN_API int attn_last_device_error(attn_stream_t stream);

/* attn_status_str -- static, human-readable name of a status code. */
ATTN_API const char* attn_status_str(int status);

/*
 * attn_set_debug -- process-wide debug switches for later launches.
 *   flags bit 0 (ATTN_DEBUG_BOUNDS): decode checks every page id against
 *                num_pages and every token against seq_len.
 *   flags bit 1 (ATTN_DEBUG_STALL): testing hook for failure detection --
 *                the kernels' load producers issue nothing, so every bounded
 *                wait runs out; the kernels release their resources, return,
 *                and attn_last_device_error() reports ATTN_ERR_TIMEOUT.  The
 *                outputs of such calls are undefined.
 *   wait_timeout_ns: limit of every bounded wait inside the kernels
 *                (0 = the default of 2 s).
 * Returns the previous flags.
 */
#define ATTN_DEBUG_BOUNDS 1
#define ATTN_DEBUG_STALL 2
ATTN_API int attn_set_debug(int flags, unsigned long long wait_timeout_ns);

/*
 * attn_last_error_message -- static, human-readable description of the last
 * host-side CUDA failure on the calling thread (the call that returned
 * ATTN_ERR_CUDA and the CUDA error string); "" if none.
 */
ATTN_API const char* attn_last_error_message(void);

/* attn_version -- ABI version of this header (currently 1). */
ATTN_API int attn_version(void);

#endif /* ATTN_SM100_H */
