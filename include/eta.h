/*
 * eta.h -- C ABI of libeta.so: fused, IO-aware exact attention forward passes for NVIDIA B200 (sm_100a).
 *
 * Every entry point computes one of the operations the reference pages define, tile by tile on the GPU,
 * without ever writing the n x n score matrix to HBM:
 *
 *   attn_fwd / attn_fwd_varlen   O = softmax(scale * Q K^T [+ causal mask]) V, plus the row logsumexp.
 *       "FlashAttention (TH)", section "ปัญหาของ Attention แบบมาตรฐาน" (the formula) and section
 *       "การคำนวณ Softmax แบบออนไลน์" (running max and exp-sum); "CANN ops-transformer 的 FlashAttention：
 *       把大模型的记忆从 32GB 压到 8GB，怎么做到的", section "FlashAttention 的解法" (online softmax, steps 1-4,
 *       only the final output written back).
 *   hstu_fwd_jagged              O = (SiLU(alpha * Q K^T) * causal_mask / n) V over packed sequences.
 *       "同样是Attention架构，为什么昇腾NPU跑HSTU时延降低10倍、显存省97%？", section "先搞懂：HSTU到底难在哪？"
 *       (the definition), "绝杀优化二：内置Mask生成" (mask generated in-kernel, masked tiles skipped) and
 *       "绝杀优化三：Jagged变长张量" (packed values + per-sequence lengths, no padding).
 *   attn_decode                  one new query per (batch, head) against a long KV cache.
 *       "AI attention complexity ledger", section "带宽账：decode 阶段的真正瓶颈"
 *       (s_j = q . k_j over all cached keys, o = sum_j p_j v_j; HBM-bound).
 *   attn_fwd_fp8                 attn_fwd on e4m3 inputs with per-tensor descales ("FlashAttention (TH)",
 *       section "FlashAttention-3").
 *   attn_decode_paged            the decode step with grouped query heads over a paged KV cache.
 *   attn_decode_noalloc          attn_decode with its scratch in the library's own device array.
 *   eta_prefill_plan, eta_prefill_sched_group, eta_status, eta_strerror, eta_set_wait_timeout_ns,
 *   eta_selftest_wait_timeout    host-side queries, the device status word and the bounded-wait limit.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Pointers named q, k, v, o, kcache, vcache, lse, cu_seqlens, kv_lens, workspace are DEVICE pointers
 *    (cudaMalloc'd or equivalent) on the current CUDA device.  The caller owns every buffer; the library
 *    allocates no device memory when called: its only device memory is the module's own static data (the
 *    status word, the prefill work counters and the allocation-free decode's scratch array).
 *  - bf16 means IEEE bfloat16 stored as 16-bit words; all tensors are contiguous, row-major, with the
 *    layouts given per call.  q, k, v, o and the caches must be 16-byte aligned.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call only enqueues work on it and
 *    returns; results are ready when the stream reaches that point.
 *  - Return value: 0 (ETA_OK) when the work was enqueued, a negative ETA_ERR_* code when the arguments
 *    are rejected on the host (nothing is enqueued then) or a CUDA launch failed.
 *  - Conditions only the device can see (a kv_lens entry outside [0, Lmax], a cu_seqlens table that is not
 *    valid for the call, a pipeline wait that ran out of time) never trap: the kernel
 *    keeps every access in bounds, records the first such condition in a device status word and carries
 *    on or returns.  Read it with eta_status().
 *  - Per-device set-up is done once and kept for the process: each kernel's shared-memory limit and
 *    register check on its first launch on a device, the allocation-free decode's scratch address, and (per
 *    host thread) the TMA descriptors of recently used buffer shapes.  A device reset (cudaDeviceReset)
 *    discards the first two; do not call the library on a device after resetting it.
 *  - Head dimension d: 64, 96 or 128 for every prefill call, 256 for softmax attention (attn_fwd,
 *    attn_fwd_varlen), 128 for the e4m3 call, 64 or 128 for decode.  The arithmetic is bf16 x bf16
 *    products accumulated in fp32 (tensor cores); softmax statistics and lse are fp32.
 */
#ifndef ETA_H_
#define ETA_H_

#include <stddef.h>

#if defined(__GNUC__)
#define ETA_API __attribute__((visibility("default")))
#else
#define ETA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Host-side error codes (negative) returned by the entry points. */
#define ETA_OK 0
#define ETA_ERR_NULL (-1)      /* a required pointer is NULL */
#define ETA_ERR_HEAD_DIM (-2)  /* d is not one the call supports (see "Head dimension" above) */
#define ETA_ERR_SHAPE (-3)     /* a size is <= 0, too large for 32-bit indexing, or inconsistent */
#define ETA_ERR_ALIGN (-4)     /* a tensor pointer is not 16-byte aligned */
#define ETA_ERR_WORKSPACE (-5) /* workspace smaller than attn_decode_workspace_size() */
#define ETA_ERR_CUDA (-6)      /* a CUDA runtime/driver call or a kernel launch failed */
#define ETA_ERR_ARG (-7)       /* a flag or scalar is out of range (o_dtype, scale, alpha, inv_n ...) */
#define ETA_ERR_DEVICE (-8)    /* the current device is not an sm_100 (B200-class) GPU */

/* Device status codes (positive) returned by eta_status(). */
#define ETA_DEV_OK 0
#define ETA_DEV_TIMEOUT 1     /* a bounded pipeline wait expired; the kernel abandoned its tile */
#define ETA_DEV_BAD_KVLEN 2   /* attn_decode: kv_lens[b] < 0 or > Lmax (clamped into range) */
#define ETA_DEV_BAD_CUSEQ 3   /* varlen/jagged: cu_seqlens not a valid offset table for the call (see attn_fwd_varlen) */
#define ETA_DEV_BAD_PAGE 4    /* attn_decode_paged: a block_table entry outside [0, num_pages) (page 0 read) */

/* Output element type selector for attn_fwd / attn_fwd_varlen. */
#define ETA_OUT_BF16 0
#define ETA_OUT_F32 1

/*
 * attn_fwd -- dense multi-head exact attention forward.
 *   q, k, v : bf16 [B, H, N, d]   (batch, heads, sequence, head dim; the pages' [batch, heads, seq_len,
 *                                  head_dim] layout, "ai6s.net FlashAttention" page, usage example)
 *   o       : [B, H, N, d], bf16 (o_dtype = ETA_OUT_BF16) or fp32 (ETA_OUT_F32)
 *   lse     : fp32 [B, H, N], natural-log logsumexp of the scaled score row, m_i + ln(sum_j e^(s_ij - m_i));
 *             may be NULL (not written)
 *   scale   : multiplies Q K^T before the softmax (1/sqrt(d) in the formula); finite and > 0
 *   causal  : 0 = every key; 1 = query i sees keys j <= i (top-left aligned, diagonal included)
 *   d       : 64, 96, 128 or 256 ("FlashAttention (TH)", section "FlashAttention-2", extends head sizes
 *             up to 256; 256 runs one 128-row Q tile per work item, see prefill_wide.cuh; a 96-element row
 *             is 1.5 swizzle chunks, the TMA zero-fills the other half chunk in shared memory)
 * Errors: ETA_ERR_NULL, ETA_ERR_HEAD_DIM, ETA_ERR_SHAPE (B,H,N <= 0 or B*H*N*d >= 2^31), ETA_ERR_ALIGN,
 *         ETA_ERR_ARG, ETA_ERR_DEVICE, ETA_ERR_CUDA.
 */
ETA_API int attn_fwd(const void *q, const void *k, const void *v, void *o, float *lse, int B, int H, int N, int d,
             float scale, int causal, int o_dtype, void *stream);

/*
 * Launches in flight (every prefill call: attn_fwd, attn_fwd_varlen, attn_fwd_fp8, hstu_fwd_jagged).
 * A prefill launch hands out its work items from a device counter.  The library holds 256 such counters per
 * device and gives each launch the next one, round-robin, when the call enqueues it; the launch's last CTA
 * returns the counter to zero.  So:
 *   - at most 256 prefill launches may be in flight on one device at a time (enqueued and not finished,
 *     over all streams); a 257th would share a counter with a launch still running, and both would skip or
 *     repeat work items;
 *   - a CUDA graph that captured a prefill call keeps that call's counter for good: do not replay one graph
 *     on two streams at once, and do not keep a replay in flight while 256 other prefill launches are
 *     enqueued after it.
 * Launches ordered on one stream never overlap, so ordinary use needs nothing.
 */

/*
 * attn_fwd_varlen -- exact attention over S packed sequences (no padding).
 *   q, k, v    : bf16 [T, H, d], T = cu_seqlens[S]; sequence s owns rows cu_seqlens[s] .. cu_seqlens[s+1]-1
 *   o          : [T, H, d] bf16 or fp32 (o_dtype);  lse: fp32 [T, H] or NULL
 *   cu_seqlens : int32 [S+1], device; cu_seqlens[0] = 0, non-decreasing
 *   max_len    : an upper bound on every sequence length (sizes the launch); T_total : cu_seqlens[S]
 *                as known to the host: the rows of q, k, v, o (and of lse) the call may touch
 *   No query attends across a sequence boundary; causal is per sequence (local indices).
 * The kernels read cu_seqlens on the device and check it against the call ("同样是Attention架构..." page,
 * section "绝杀优化三：Jagged变长张量": the offsets are the whole state of a jagged tensor).  A sequence whose
 * offsets are negative or decreasing, longer than max_len, or end past T_total is skipped (nothing of it is
 * read or written, so no access leaves [0, T_total)); that, and a first offset other than 0 or a last offset
 * other than T_total (sequences inside [0, T_total) are still computed), record ETA_DEV_BAD_CUSEQ.
 * Zero-length sequences produce nothing.  Errors as attn_fwd, plus device status ETA_DEV_BAD_CUSEQ.
 */
ETA_API int attn_fwd_varlen(const void *q, const void *k, const void *v, void *o, float *lse, const int *cu_seqlens,
                    int S, int max_len, int T_total, int H, int d, float scale, int causal, int o_dtype,
                    void *stream);

/*
 * attn_fwd_fp8 -- attn_fwd with 8-bit inputs ("FlashAttention (TH)", section "FlashAttention-3": FP8 support).
 * The pages give no scaling recipe; this one is per tensor: the caller passes q8, k8, v8 holding e4m3 values
 * (torch.float8_e4m3fn, one byte each, [B, H, N, d]) and positive descale factors with Q = q8 * q_descale,
 * K = k8 * k_descale, V = v8 * v_descale.  Then
 *   s_ij = scale * q_descale * k_descale * (q8_i . k8_j)   (exact products, fp32 accumulation),
 *   o_i  = v_descale * sum_j P8_ij v8_j / sum_j P_ij,  P_ij = e^(s_ij - m_i) as fp32, P8 its e4m3 rounding
 *          (nearest; the P . V product runs on e4m3 operands), lse_i as in attn_fwd.
 *   d must be 128 (a row is one 128-byte span); o bf16 or fp32 (o_dtype); lse fp32 or NULL.
 * Errors as attn_fwd; ETA_ERR_HEAD_DIM for d != 128, ETA_ERR_ARG for a non-finite or non-positive descale.
 */
ETA_API int attn_fwd_fp8(const void *q, const void *k, const void *v, void *o, float *lse, int B, int H, int N,
                         int d, float scale, float q_descale, float k_descale, float v_descale, int causal,
                         int o_dtype, void *stream);

/*
 * hstu_fwd_jagged -- HSTU pointwise attention over S packed sequences:
 *   x_ij = alpha * q_i . k_j ;  p_ij = silu(x_ij) * inv_n  for j <= i (local indices), 0 otherwise ;
 *   o_i = sum_j p_ij v_j.
 *   q, k, v : bf16 [T, H, d]; o : bf16 [T, H, d]; cu_seqlens, S, max_len, T_total as attn_fwd_varlen.
 *   alpha   : the page's alpha (finite); inv_n : 1/n of the page's "x *= mask / n" (finite, > 0).
 * There is no softmax, no running max and no lse.  Errors as attn_fwd_varlen.
 */
ETA_API int hstu_fwd_jagged(const void *q, const void *k, const void *v, void *o, const int *cu_seqlens, int S,
                    int max_len, int T_total, int H, int d, float alpha, float inv_n, void *stream);

/*
 * attn_decode_workspace_size -- bytes of device workspace attn_decode needs for these sizes
 * (split-KV partial outputs and their logsumexps).  Returns 0 for invalid sizes.
 */
ETA_API size_t attn_decode_workspace_size(int B, int H, int Lmax, int d);

/*
 * attn_decode -- one decode step: for each (b, h), the single query q[b,h,:] attends (non-causally) to the
 * cached keys/values rows 0 .. kv_lens[b]-1.
 *   q         : bf16 [B, H, d]
 *   kcache    : bf16 [B, H, Lmax, d];  vcache : bf16 [B, H, Lmax, d]; rows >= kv_lens[b] are never read
 *   kv_lens   : int32 [B], device, each in [0, Lmax]; a zero length gives o = 0, lse = -inf
 *   o         : bf16 [B, H, d];  lse : fp32 [B, H] or NULL
 *   workspace : device buffer of at least attn_decode_workspace_size(B, H, Lmax, d) bytes, 16-byte
 *               aligned, owned by the caller; its contents need no initialisation and are scratch.
 * The cache is split along the sequence into chunks processed by independent CTAs (split-KV); the chunks'
 * partial results are merged with logsumexp weights, which is exact.
 * Errors as attn_fwd, plus ETA_ERR_WORKSPACE and device status ETA_DEV_BAD_KVLEN.
 */
ETA_API int attn_decode(const void *q, const void *kcache, const void *vcache, const int *kv_lens, void *o, float *lse,
                int B, int H, int Lmax, int d, float scale, void *workspace, size_t workspace_bytes,
                void *stream);

/*
 * attn_decode_paged_workspace_size -- bytes of device workspace attn_decode_paged needs (split-KV partials of
 * every query head).  Returns 0 for invalid sizes.
 */
ETA_API size_t attn_decode_paged_workspace_size(int B, int Hq, int max_pages, int page_size, int d);

/*
 * attn_decode_paged -- one decode step with grouped query heads over a paged KV cache.  The decode step of
 * "AI attention complexity ledger", section "带宽账：decode 阶段的真正瓶颈", with the two cache-side changes
 * the pages name: key/value heads shared by groups of query heads (the same section's GQA route for
 * shrinking the KV cache; "FlashAttention (TH)", section "FlashAttention-2": MQA) and a cache held in fixed
 * pages reached through a page table (the ops-transformer page: KV-cache management, PagedAttention).
 * For each b and query head hq, with G = Hq / Hkv and kv head g = hq / G:
 *   s_j = scale * q[b,hq,:] . K_j,  o[b,hq,:] = sum_j softmax(s)_j V_j,  j = 0 .. kv_lens[b]-1,
 * where row j of sequence b is row (j % page_size) of page block_table[b][j / page_size], kv head g.
 *   q           : bf16 [B, Hq, d]
 *   k_pages     : bf16 [num_pages, Hkv, page_size, d]  (page pool; each (page, kv head) is one contiguous
 *                 page_size x d block); v_pages : same layout
 *   block_table : int32 [B, max_pages], device; entries for pages 0 .. ceil(kv_lens[b]/page_size)-1 must lie
 *                 in [0, num_pages) (others are never read); sequences may share pages
 *   kv_lens     : int32 [B], device, each in [0, max_pages * page_size]; zero gives o = 0, lse = -inf
 *   o           : bf16 [B, Hq, d];  lse : fp32 [B, Hq] or NULL
 *   Hq % Hkv == 0 and Hq / Hkv <= 16; page_size in {16, 32, 64, 128, 256}; d in {64, 128};
 *   num_pages * Hkv, max_pages * page_size and B * max_pages below 2^31.
 *   workspace   : device buffer of at least attn_decode_paged_workspace_size(B, Hq, max_pages, page_size, d)
 *                 bytes, 16-byte aligned, owned by the caller, scratch.
 * Rows past kv_lens[b] inside the last page are never used (whatever they hold).  The cache is split along
 * the sequence (split-KV) and the splits merged with logsumexp weights, which is exact.
 * Errors: ETA_ERR_NULL, ETA_ERR_HEAD_DIM, ETA_ERR_SHAPE, ETA_ERR_ALIGN, ETA_ERR_ARG, ETA_ERR_WORKSPACE,
 * ETA_ERR_DEVICE, ETA_ERR_CUDA; device status ETA_DEV_BAD_KVLEN (length clamped into range) and
 * ETA_DEV_BAD_PAGE (an out-of-range page number; page 0 is read in its place).
 */
ETA_API int attn_decode_paged(const void *q, const void *k_pages, const void *v_pages, const int *block_table,
                              const int *kv_lens, void *o, float *lse, int B, int Hq, int Hkv, int num_pages,
                              int page_size, int max_pages, int d, float scale, void *workspace,
                              size_t workspace_bytes, void *stream);

/*
 * attn_decode_noalloc -- the same decode step as attn_decode, for callers that cannot allocate device memory
 * when they call: for example a plugin running inside a host engine that owns all device memory and forbids
 * allocation in its enqueue step, or a latency-critical loop that cannot afford cudaMalloc's implicit
 * device synchronisation.  It takes no workspace argument: the split-KV partial results go to a fixed
 * scratch array of ETA_NOALLOC_SCRATCH_BYTES that the library holds in device memory (one copy on every GPU
 * that loads the library, kept until the process exits).  The pages have no counterpart; it is an
 * interface convenience around the decode kernels.
 *   Arguments, layouts and results are exactly those of attn_decode (minus workspace / workspace_bytes).
 *   The first call on a device, with that device current, looks up the scratch array's device address
 *   (cudaGetSymbolAddress); make that first call before any stream capture.  No call allocates or frees
 *   memory.
 *   Returns ETA_ERR_WORKSPACE, and enqueues nothing, when attn_decode_workspace_size(B, H, Lmax, d) exceeds
 *   ETA_NOALLOC_SCRATCH_BYTES; other errors as attn_decode.
 *   All calls on a device share the one scratch array, which keeps the last call's contents (every value a
 *   call reads is written earlier by that same call, so nothing needs clearing).  Calls whose GPU work
 *   overlaps -- on different streams, or from different host threads -- race on it: serialise them.
 */
#define ETA_NOALLOC_SCRATCH_BYTES (8u << 20)
ETA_API int attn_decode_noalloc(const void *q, const void *kcache, const void *vcache, const int *kv_lens, void *o,
                                float *lse, int B, int H, int Lmax, int d, float scale, void *stream);

/*
 * eta_prefill_plan -- the work decomposition a prefill call would launch on a GPU with `sms` SMs (host
 * logic only: no GPU is touched).  kind: 0 = attn_fwd / attn_fwd_fp8, 1 = attn_fwd_varlen,
 * 2 = hstu_fwd_jagged (always causal).  units = B*H (dense) or S*H (packed); rows = N (dense) or max_len.
 * A work item is 256 query rows (two 128-row Q tiles; 128 rows at d = 256) of one unit.  Outputs (each may be
 * NULL): *items = work items; *whole = items run whole, the other items - whole are each run as two split
 * halves (one Q tile, its key tiles divided between the CTA's two softmax warpgroups); *ctas = CTAs of the
 * persistent grid.  The split rule: non-causal launches whose last wave is at most half full split those
 * last items; causal launches with no more items than SMs, and non-causal ones with at most half as many,
 * split every item; HSTU and d = 256 never split.
 * Returns 0, or ETA_ERR_HEAD_DIM / ETA_ERR_SHAPE / ETA_ERR_ARG as the planned call would.
 */
ETA_API int eta_prefill_plan(int kind, long long units, long long rows, int d, int causal, int sms,
                             long long *items, long long *whole, int *ctas);

/*
 * eta_prefill_sched_group -- how many (batch, head) units a dense prefill launch (attn_fwd, attn_fwd_fp8)
 * schedules together (host logic only).  Items are handed out group by group, and inside a group the latest
 * row block of every unit first, so that the K and V of a group (2 * rows * d * elt_bytes bytes per unit,
 * kept within 32 MiB) stay in L2 while its row blocks run and are read from HBM about once.  rows = N;
 * elt_bytes = 2 (bf16) or 1 (e4m3).  Returns a count in [1, units], or ETA_ERR_SHAPE.
 */
ETA_API long long eta_prefill_sched_group(long long units, long long rows, int d, int elt_bytes);

/*
 * eta_status -- synchronises `stream`, returns the device status word of the current device
 * (ETA_DEV_*; the first condition recorded since the last call) and clears it.  Returns ETA_ERR_CUDA if
 * the synchronisation or the copy failed.
 */
ETA_API int eta_status(void *stream);

/* eta_strerror -- a static, human-readable description of any ETA_* code. */
ETA_API const char *eta_strerror(int code);

/*
 * eta_set_wait_timeout_ns -- upper bound, in nanoseconds of %globaltimer, on every pipeline wait inside
 * the kernels (default 2e9 = 2 s).  A wait that runs out records ETA_DEV_TIMEOUT and the kernel returns.
 * Values <= 0 restore the default.  Applies to launches made after the call.
 */
ETA_API void eta_set_wait_timeout_ns(long long ns);

/*
 * eta_selftest_wait_timeout -- launches one CTA that waits on a pipeline barrier nothing will ever
 * complete, under the current bounded-wait limit, so that a test can check the limit and the status word
 * without faulting or hanging the GPU.  Returns 0 when enqueued; the caller then reads eta_status().
 */
ETA_API int eta_selftest_wait_timeout(void *stream);

#ifdef __cplusplus
}
#endif

#endif /* ETA_H_ */
