/*
 * gqa_paged.h -- C ABI of libgqa_paged.so: grouped-query attention (GQA) over a paged
 * KV cache, for NVIDIA B200 (sm_100a).
 *
 * The operation (sources by page title and section):
 *   - GQA: Hq query heads form Hk groups of g = Hq/Hk consecutive heads; every head of a
 *     group reads the same K/V head, kv head = h / g
 *     ("TensorRT对Grouped Query Attention的支持进展", sections
 *     "技术演进背景：从MHA到GQA的必然选择" and "图优化与算子融合", RepeatKV).
 *   - Paged KV cache: each sequence's keys and values live in fixed-size pages of a pool
 *     owned by the caller; a per-sequence page table maps logical page p to a physical
 *     page ("TensorRT-LLM与TensorRT核心差异解析", section 4.2.2 PageAttention;
 *     "TensorRT对Grouped Query Attention的支持进展", section "动态形状与KV Cache管理":
 *     the caller keeps the pool and passes physical page indices on every call).
 *   - Fused attention: softmax(scale * q K^T) V computed tile by tile on chip, only the
 *     output written back ("TensorRT-LLM与TensorRT核心差异解析", section 4.2.1).
 *   - PackGQA and NumSplits ("解锁GQA性能潜力：从批量大小敏感性到高效优化实践",
 *     section "核心参数调优：PackGQA与NumSplits的协同舞蹈"): all query heads of a group
 *     share one thread block so each KV page is read once; long contexts are split
 *     across thread blocks and merged by log-sum-exp (lse_combine).
 *   - Chunked prefill ("TensorRT对Grouped Query Attention的支持进展", section
 *     "与动态批处理协同").
 *   - FP8 KV ("解锁GQA性能潜力…", section "实践验证：从理论到落地的性能跃迁").
 *
 * Common conventions for every call:
 *   - Every data pointer is a DEVICE pointer owned by the caller.  The library keeps
 *     no reference after the call returns and allocates no device memory; scratch
 *     space comes from the caller's `workspace`.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; 0 = legacy default stream).
 *   - Return value: GQA_OK (0) when the work was enqueued; a negative gqa_status_t when
 *     host-side validation failed (then nothing was enqueued) or a launch failed.
 *   - Device-side errors (a page-table entry outside [0, num_pages), a bounded wait that
 *     ran out) are recorded in an int32 error word at the start of `workspace` and read
 *     and cleared by gqa_get_error().  A workspace must be zero-filled once before its
 *     first use; after that the library only ever sets the word and gqa_get_error()
 *     clears it.
 *   - Layouts are row-major (C order).  KV pools are [num_pages][Hk][page_size][head_dim]
 *     ("HND": each (page, kv head) block is one contiguous run).  q and out are bf16.
 *   - Sequence lengths count the current token(s): the new K/V are in the cache, written
 *     by the caller or by gqa_paged_append_kv().  No other call writes the cache.
 *   - Page-table entries at or beyond ceil(seq_len / page_size) are never read; entries
 *     may repeat across and within sequences (shared prefix pages).
 *   - A sequence of length 0 yields output 0 and lse = -inf.
 *   - The device arrays must not change until the enqueued work has finished.
 */
#ifndef GQA_PAGED_H_
#define GQA_PAGED_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GQA_OK = 0,
    GQA_ERR_NULL = -1,      /* a required pointer is NULL */
    GQA_ERR_SHAPE = -2,     /* unsupported or inconsistent sizes (Hq % Hk, head_dim, page_size, ...) */
    GQA_ERR_DTYPE = -3,     /* unknown kv_dtype, or fp8 without scales, or fp8 with head_dim != 128 */
    GQA_ERR_SPLITS = -4,    /* num_splits outside 0..GQA_MAX_SPLITS */
    GQA_ERR_WORKSPACE = -5, /* workspace NULL, smaller than the *_workspace_size() value, or not 256-byte aligned */
    GQA_ERR_LAUNCH = -6,    /* a CUDA launch or driver call failed */
    GQA_ERR_BAD_PAGE = -7,  /* (device) a page-table entry read was outside [0, num_pages) */
    GQA_ERR_TIMEOUT = -8,   /* (device) a bounded pipeline wait ran out; the kernel gave up */
    GQA_ERR_ALIGN = -9      /* a pointer is not 16-byte aligned */
} gqa_status_t;

typedef enum {
    GQA_KV_BF16 = 0,     /* k_pages / v_pages hold bf16 */
    GQA_KV_FP8_E4M3 = 1  /* k_pages / v_pages hold OCP e4m3 bytes; value = code * scale[page][kv head] */
} gqa_kv_dtype_t;

#define GQA_MAX_SPLITS 64
/* num_splits value that asks for the balanced persistent schedule whatever the problem
 * size (B <= 2048), for comparison sweeps; 0 lets the measured table decide. */
#define GQA_SPLITS_BALANCED (-1)

/*
 * Bytes of workspace gqa_paged_decode() needs for the same B, heads, head_dim, page_size,
 * longest context (pt_stride * page_size), kv_dtype and num_splits.  Layout: a 256-byte
 * header holding the device error word, then
 *   num_splits = 0, B <= 2048 (balanced schedule): int32 merge counters [B*Hq] (rounded
 *     up to 256 bytes) and the merge pieces, 2 per worker of the largest grid
 *     (160 SMs x 2 CTAs x 4 workers), each min(Hq/Hk, 16) x (head_dim + 1) fp32;
 *   split schedule with S > 1: o_part fp32 [S][B*Hq][head_dim] and lse_part fp32 [S][B*Hq].
 */
size_t gqa_paged_decode_workspace_size(int B, int Hq, int Hk, int head_dim, int page_size,
                                       int max_seq_len, int kv_dtype, int num_splits);

/*
 * Kernels one gqa_paged_decode() call with these arguments launches on the current
 * device: 1, or 2 when a second kernel merges partial results (split schedule with
 * S > 1: lse_combine; balanced schedule when its units average more than 8 workers
 * each, e.g. a few long sequences: the kernel that merges the pieces of cut units).
 * Returns 0 for sizes gqa_paged_decode() rejects.  Host only; launches nothing.
 */
int gqa_paged_decode_kernel_launches(int B, int Hq, int Hk, int head_dim, int page_size,
                                     int max_seq_len, int kv_dtype, int num_splits,
                                     int pack_gqa);

/*
 * The split schedule's measured fastest split count for B sequences of Hk kv heads and
 * context max_seq_len: a table measured on one B200 over units (B * Hk, scaled to this
 * device's SM count) and context, for bf16 and e4m3 KV, nearest entry in log scale.
 * gqa_paged_decode() uses it with num_splits = 0 when B is above the balanced schedule's
 * limit (2048).
 */
int gqa_pick_splits(int B, int Hk, int max_seq_len, int page_size, int kv_dtype);

/*
 * Decode: one new query token per sequence attends to all seq_lens[b] tokens of its
 * paged history.  For sequence b and query head h (kv head j = h / (Hq/Hk)):
 *   s_t = scale * <q[b][h], K_b[t]>,  out[b][h] = sum_t softmax(s)_t V_b[t],
 *   lse[b][h] = ln sum_t exp(s_t)
 * with K_b[t] = k_pages[page_table[b][t / page_size]][j][t % page_size].
 *
 *   q          bf16 [B][Hq][head_dim]
 *   k_pages,
 *   v_pages    [num_pages][Hk][page_size][head_dim] of kv_dtype; 16-byte aligned
 *   k_scale,
 *   v_scale    fp32 [num_pages][Hk] for GQA_KV_FP8_E4M3; ignored (may be NULL) for bf16
 *   page_table int32 [B][pt_stride]; pt_stride >= ceil(max seq_len / page_size)
 *   seq_lens   int32 [B], each in [0, pt_stride * page_size]
 *   Hq % Hk == 0; head_dim in {64, 128}; page_size in {16, 32, 64}
 *   scale      softmax scale (commonly 1/sqrt(head_dim))
 *   num_splits 0 = automatic: for B <= 2048 a balanced persistent schedule: all
 *              (sequence, kv head) tiles of 16 tokens are laid end to end and shared
 *              equally by the workers of a fixed grid, and units cut between workers are
 *              merged by log-sum-exp inside the same launch (by a second kernel where the
 *              units average more than 8 workers each) -- except for the small
 *              problems (a few sequences of short context pt_stride*page_size) where the
 *              split schedule measured faster, which run splits with the measured count;
 *              for larger B, splits with the count gqa_pick_splits gives.
 *              GQA_SPLITS_BALANCED (-1): the balanced schedule for any B <= 2048.
 *              1..GQA_MAX_SPLITS: contiguous page-aligned ranges of ceil(np / num_splits)
 *              pages (np = ceil(seq_len / page_size)), merged with lse_combine on the
 *              same stream
 *   pack_gqa   1 (default): all heads of a group in one thread block, each KV page read
 *              once; 0: one query head per thread block (for comparison sweeps only)
 *   out        bf16 [B][Hq][head_dim]
 *   lse        fp32 [B][Hq] natural-log log-sum-exp, or NULL
 *   workspace  >= gqa_paged_decode_workspace_size(...) bytes, 256-byte aligned, zeroed
 *              before first use.  The balanced schedule keeps one merge counter per
 *              (sequence, head) in it, back to zero at the end of every launch; after a
 *              device-side error (see gqa_get_error) zero the workspace again.
 * The balanced schedule's kernel is launched with programmatic stream serialization: its
 * CTAs may start (shared-memory set-up only) while the previous kernel on `stream` is
 * still running, and read or write no global memory until that kernel has completed.
 * Stream order is therefore kept as for an ordinary launch.
 */
int gqa_paged_decode(const void *q, const void *k_pages, const void *v_pages,
                     const float *k_scale, const float *v_scale, int kv_dtype,
                     const int32_t *page_table, int pt_stride, const int32_t *seq_lens, int B,
                     int Hq, int Hk, int head_dim, int page_size, int num_pages, float scale,
                     int num_splits, int pack_gqa, void *out, float *lse, void *workspace,
                     size_t workspace_bytes, cudaStream_t stream);

/*
 * Decode over this rank's share of each sequence's history, for a sequence whose pages are
 * spread over several GPUs: every GPU computes the attention of the new query token over
 * the tokens it holds, the GPUs exchange these partial results, and each merges them with
 * lse_combine() ("FasterTransformer source tour", section 6.1: splitting a context too
 * long for one device across devices; the merge is the NumSplits log-sum-exp merge of
 * "解锁GQA性能潜力：从批量大小敏感性到高效优化实践", section
 * "核心参数调优：PackGQA与NumSplits的协同舞蹈").
 *
 * Arguments and checks are gqa_paged_decode()'s: page_table / seq_lens describe the
 * tokens THIS call covers (its rows of the page table and the number of those tokens per
 * sequence, 0 for a sequence with none here).  The results are written in fp32 instead of
 * bf16, in the form lse_combine() takes for one split:
 *   o_part    fp32 [B][Hq][head_dim]: softmax-normalised attention over the covered tokens
 *             (0 for a sequence with none), 16-byte aligned
 *   lse_part  fp32 [B][Hq]: natural-log log-sum-exp of the covered scores (-inf for a
 *             sequence with none); required (NULL gives GQA_ERR_NULL)
 * Stacking the o_part / lse_part of R such calls (R ranks, or R disjoint page ranges) as
 * [R][B*Hq][head_dim] / [R][B*Hq] and passing them to lse_combine(num_splits = R) gives
 * the decode over all their tokens.  Workspace: gqa_paged_decode_workspace_size() with
 * the same arguments.
 */
int gqa_paged_decode_partial(const void *q, const void *k_pages, const void *v_pages,
                             const float *k_scale, const float *v_scale, int kv_dtype,
                             const int32_t *page_table, int pt_stride, const int32_t *seq_lens,
                             int B, int Hq, int Hk, int head_dim, int page_size, int num_pages,
                             float scale, int num_splits, int pack_gqa, float *o_part,
                             float *lse_part, void *workspace, size_t workspace_bytes,
                             cudaStream_t stream);

/*
 * Largest scratch gqa_paged_decode_static_scratch() can use: its fixed array's size.
 */
#define GQA_STATIC_SCRATCH_BYTES (16u << 20)

/*
 * gqa_paged_decode() without a workspace argument.  The pages have no counterpart: this is
 * an interface convenience, and the computation is exactly gqa_paged_decode()'s.
 *
 * Who it is for: callers that cannot allocate device memory where they run decode.
 * Examples are an inference-engine plugin whose enqueue step may not allocate, a loop
 * with a real-time budget that forbids allocation after start-up, and a host whose
 * device memory is all handed out by another allocator.  Such callers cannot create and
 * own the workspace that gqa_paged_decode() needs for its split partials.
 *
 * How: the scratch (error word, then o_part / lse_part) lives in one fixed
 * GQA_STATIC_SCRATCH_BYTES array compiled into this library (a `static __device__`
 * array).  Every GPU that loads the library holds the array until the process exits.
 * Nothing is allocated: no cudaMalloc, cudaFree or allocating library routine is called.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current) and caches it.  Make that first
 *     call before any stream capture.
 *   - Every call on a device shares the one array, which keeps the last call's contents.
 *     Each call clears the error word (an async memset on `stream`) and fully rewrites
 *     the partials it uses.  Calls that overlap on the GPU (other streams, other threads)
 *     race on the array: serialise them.
 *   - Device-side errors (out-of-range page entries, a bounded wait that ran out) are
 *     recorded in the array's error word but cannot be read back through this entry
 *     point.  Use gqa_paged_decode() with a workspace when those reports are needed.
 *   - The cached address belongs to the device's context as it was at the first call:
 *     calls after cudaDeviceReset() on that device are not supported.
 *
 * Arguments are gqa_paged_decode()'s, minus workspace / workspace_bytes.  Returns what
 * gqa_paged_decode() returns; its argument checks run first, so a call it rejects
 * enqueues nothing.  Also returns GQA_ERR_WORKSPACE, with nothing enqueued, when the call
 * needs more than GQA_STATIC_SCRATCH_BYTES of scratch, i.e. when
 * gqa_paged_decode_workspace_size(B, Hq, Hk, head_dim, page_size,
 * pt_stride * page_size, kv_dtype, num_splits) exceeds it.  Lower num_splits or the
 * batch to fit.  One case never fits with num_splits = 0: groups of more than 8 query
 * heads per kv head at head_dim 128 (the balanced schedule's merge pieces alone take
 * about 21 MB); pass num_splits >= 1 for those.
 */
int gqa_paged_decode_static_scratch(const void *q, const void *k_pages, const void *v_pages,
                                    const float *k_scale, const float *v_scale, int kv_dtype,
                                    const int32_t *page_table, int pt_stride,
                                    const int32_t *seq_lens, int B, int Hq, int Hk,
                                    int head_dim, int page_size, int num_pages, float scale,
                                    int num_splits, int pack_gqa, void *out, float *lse,
                                    cudaStream_t stream);

/*
 * Bytes of workspace gqa_paged_prefill() needs for total_q query tokens: the 256-byte
 * error-word header, then the launch plan (the count and one int per work item, a work
 * item being two query tiles of one sequence: at most one per query token), rounded up to
 * 256 bytes.  Hq and head_dim are accepted for symmetry with the decode call.
 */
size_t gqa_paged_prefill_workspace_size(int total_q, int Hq, int head_dim);

/*
 * Causal chunked prefill: sequence b appends Lq_b = cu_q[b+1] - cu_q[b] new query tokens
 * after a paged prior context; the chunk's K/V are already the last Lq_b of the
 * seq_lens[b] cached tokens.  Query row i of sequence b sits at position
 * pos = seq_lens[b] - Lq_b + i and, when causal, attends to tokens 0..pos (all
 * seq_lens[b] tokens when causal == 0).
 *
 *   q          bf16 [total_q][Hq][head_dim], rows of sequence b at cu_q[b] .. cu_q[b+1]-1
 *   cu_q       int32 [B+1], cu_q[0] = 0, nondecreasing, cu_q[B] = total_q,
 *              cu_q[b+1] - cu_q[b] <= max_q_len and <= seq_lens[b]
 *   k_pages, v_pages, page_table, pt_stride, seq_lens: as for decode (bf16 KV only)
 *   head_dim   64 or 128; page_size in {16, 32, 64}; Hq / Hk <= 128; scale > 0
 *   out        bf16 [total_q][Hq][head_dim];  lse fp32 [total_q][Hq] or NULL
 *   workspace  >= gqa_paged_prefill_workspace_size(...) bytes, zeroed before first use
 */
int gqa_paged_prefill(const void *q, const int32_t *cu_q, const void *k_pages,
                      const void *v_pages, const int32_t *page_table, int pt_stride,
                      const int32_t *seq_lens, int B, int Hq, int Hk, int head_dim,
                      int page_size, int num_pages, float scale, int causal, int total_q,
                      int max_q_len, void *out, float *lse, void *workspace,
                      size_t workspace_bytes, cudaStream_t stream);

/*
 * Log-sum-exp merge of split attention results ("解锁GQA性能潜力…", NumSplits).  For
 * every row r:  M = max_s lse_part[s][r],  w_s = exp(lse_part[s][r] - M),
 *   out[r] = sum_s w_s o_part[s][r] / sum_s w_s,   lse[r] = M + ln sum_s w_s.
 * Rows whose splits are all empty (lse = -inf) give out = 0, lse = -inf.
 *
 *   o_part   fp32 [num_splits][rows][head_dim], each split's output already normalised
 *   lse_part fp32 [num_splits][rows], natural log
 *   out      bf16 [rows][head_dim];  lse fp32 [rows] or NULL
 *   1 <= num_splits <= GQA_MAX_SPLITS, head_dim in {64, 128}
 */
int lse_combine(const float *o_part, const float *lse_part, int num_splits, int rows,
                int head_dim, void *out, float *lse, cudaStream_t stream);

/*
 * KV append: writes each sequence's new token into the paged cache, the step before decode
 * (the fused decoder step of "FasterTransformer source tour" counts this write among its
 * three global accesses).  seq_lens[b] already counts the new token, so token L_b - 1 of
 * sequence b goes to page page_table[b][(L_b - 1) / page_size], slot (L_b - 1) % page_size,
 * for every kv head j:
 *   bf16 pools:  k_pages[...][j][slot][:] = k_new[b][j][:] (bits copied), same for v.
 *   e4m3 pools:  a token that opens a page (slot 0) sets k_scale[page][j] = absmax / 448
 *                (fp32; 1 for an all-zero token), a later token keeps the page's scale;
 *                each element is stored as e4m3(x / scale), the fp32 quotient rounded to
 *                nearest even and saturated at +-448.  The same for v.
 * Sequences with seq_lens[b] = 0 append nothing.
 *
 *   k_new, v_new  bf16 [B][Hk][head_dim]
 *   k_pages, v_pages, page_table, seq_lens, page sizes: as for gqa_paged_decode()
 *   k_scale, v_scale  fp32 [num_pages][Hk], read and written for GQA_KV_FP8_E4M3
 *   workspace   >= 256 bytes, 256-byte aligned; its error word records a page-table
 *               entry or seq_len out of range (that token is not written)
 * Two sequences whose new tokens fall on the same (page, slot) race.
 */
int gqa_paged_append_kv(const void *k_new, const void *v_new, void *k_pages, void *v_pages,
                        float *k_scale, float *v_scale, int kv_dtype, const int32_t *page_table,
                        int pt_stride, const int32_t *seq_lens, int B, int Hk, int head_dim,
                        int page_size, int num_pages, void *workspace, cudaStream_t stream);

/*
 * gqa_paged_append_kv() then gqa_paged_decode() on the same stream: the new token of every
 * sequence is written into its page, then attended to with the rest of the history.
 * Arguments are the two calls'; the decode's checks run first, so a rejected call
 * changes nothing.  The decode kernel starts its set-up while the append kernel finishes
 * and reads the cache only after it has completed.
 */
int gqa_paged_append_decode(const void *q, const void *k_new, const void *v_new, void *k_pages,
                            void *v_pages, float *k_scale, float *v_scale, int kv_dtype,
                            const int32_t *page_table, int pt_stride, const int32_t *seq_lens,
                            int B, int Hq, int Hk, int head_dim, int page_size, int num_pages,
                            float scale, int num_splits, int pack_gqa, void *out, float *lse,
                            void *workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Copy-out of the paged cache into contiguous per-sequence storage, bit for bit:
 *   k_out[cu_kv[b] + t][j][:] = k_pages[page_table[b][t / page_size]][j][t % page_size][:]
 * and the same for v, for t < seq_lens[b].  elem_bytes is 2 (bf16) or 1 (fp8); bytes
 * are copied, never interpreted.  A check of the page-table indirection on its own.
 *
 *   cu_kv    int64 [B+1] output row offsets (cu_kv[b+1] - cu_kv[b] = seq_lens[b])
 *   k_out, v_out  [cu_kv[B]][Hk][head_dim] elements
 * Page-table entries outside [0, num_pages) are not read; their rows are left unwritten
 * and the call still succeeds (use the decode error word to detect bad tables).
 */
int gqa_paged_gather(const void *k_pages, const void *v_pages, const int32_t *page_table,
                     int pt_stride, const int32_t *seq_lens, const int64_t *cu_kv, int B,
                     int Hk, int head_dim, int page_size, int num_pages, int elem_bytes,
                     void *k_out, void *v_out, cudaStream_t stream);

/* ---------------------------------------------------------------------------------------
 * Page-level top-K sparse decode: the decode stage of RocketKV as
 * "TensorRT-LLM 如何用 sparse_attention_config 配置 Sparse Attention 降低长上下文推理开销"
 * (RocketKV configuration section) configures it: an auxiliary KT cache scores every page
 * of a sequence, and the decode attends to the `topk` best pages plus the pages holding the
 * last `window` tokens (the page's window_size), skipping the rest.  The page leaves the
 * KT cache and the score unstated; this library reads them as follows.
 *   - KT entry of (page, kv head): the element-wise minimum and maximum of the page's key
 *     vectors over its valid tokens.  kt: bf16 [num_pages][Hk][head_dim][2], (min, max)
 *     per dim, 16-byte aligned, owned by the caller (like the KV pools).
 *   - Score of a page for kv head j: over the g query heads h of the group,
 *     sum_h sum_d max(q[h][d] * min_d, q[h][d] * max_d), the largest q.k over the box
 *     [min, max] (an upper bound of q.k for every key of the page).  fp32, d ascending
 *     per head, then heads ascending (every product of two bf16 values is exact in fp32).
 *   - Selection per (sequence, kv head): the pages holding any of the last `window` tokens
 *     (none when window = 0), plus the `topk` highest-scoring earlier pages, equal scores
 *     going to the lower logical page; all earlier pages when there are at most `topk`.
 *     The selection unit is one cache page (the page's sparse page_size, a power of two,
 *     taken equal to page_size), and every query channel is used (the page's topr =
 *     head_dim).
 *   - Attention: softmax attention of every query head over the tokens of its kv head's
 *     chosen pages, computed by the decode kernels of gqa_paged_decode().
 * bf16 pools only; head_dim in {64, 128}; Hq / Hk <= 16; pt_stride <= 16384.
 * ------------------------------------------------------------------------------------- */

/*
 * KT entries of every page the sequences reference: for sequence b and logical page
 * p < ceil(seq_lens[b] / page_size), the min / max over the page's
 * min(page_size, seq_lens[b] - p * page_size) valid tokens.  Entries of unreferenced pages
 * are not written.  A page referenced by several sequences must hold the same number of
 * valid tokens in each (shared prefix pages are full pages); they then write equal values.
 * workspace: >= 256 bytes, 256-byte aligned; its error word records page-table entries or
 * sequence lengths out of range.
 */
int gqa_paged_kt_build(const void *k_pages, const int32_t *page_table, int pt_stride,
                       const int32_t *seq_lens, int B, int Hk, int head_dim, int page_size,
                       int num_pages, void *kt, void *workspace, cudaStream_t stream);

/*
 * KT update for the token gqa_paged_append_kv() writes (position seq_lens[b] - 1): a token
 * that opens a page (slot 0) sets the page's entry to (k, k), a later one takes the
 * element-wise min / max with it.  k_new bf16 [B][Hk][head_dim].  After appends, the
 * entries equal gqa_paged_kt_build()'s for the grown sequences.
 */
int gqa_paged_kt_append(const void *k_new, const int32_t *page_table, int pt_stride,
                        const int32_t *seq_lens, int B, int Hk, int head_dim, int page_size,
                        int num_pages, void *kt, void *workspace, cudaStream_t stream);

/*
 * Entries per row of the chosen-page table: min(pt_stride, topk + window pages), the
 * window touching at most ceil(window / page_size) + 1 pages.  0 for invalid arguments.
 */
int gqa_paged_sparse_table_stride(int pt_stride, int page_size, int topk, int window);

/* Workspace of gqa_paged_sparse_select(): the error-word header, then the page scores
 * (one 32-bit key per (sequence, kv head, page)). */
size_t gqa_paged_sparse_select_workspace_size(int B, int Hk, int pt_stride);

/*
 * The selection alone.  For row r = b * Hk + j (sequence b, kv head j):
 *   sel_table int32 [B*Hk][sel_stride]: the chosen pages in ascending logical order, each
 *             as physical page * Hk + j (the (page, kv head) block's index when the pools
 *             are seen as [num_pages * Hk][1][page_size][head_dim])
 *   sel_lens  int32 [B*Hk]: tokens in the chosen pages
 *   sel_pages int32 [B*Hk][sel_stride] or NULL: the chosen logical page indices
 *   sel_stride >= gqa_paged_sparse_table_stride(pt_stride, page_size, topk, window)
 * workspace: >= gqa_paged_sparse_select_workspace_size(B, Hk, pt_stride) bytes, 256-byte
 * aligned, zeroed before first use (error word, then the scores between the two kernels:
 * one scores pages in chunks of 64 over a (chunk, kv head, sequence) grid, one picks).
 */
int gqa_paged_sparse_select(const void *q, const void *kt, const int32_t *page_table,
                            int pt_stride, const int32_t *seq_lens, int B, int Hq, int Hk,
                            int head_dim, int page_size, int num_pages, int topk, int window,
                            int32_t *sel_table, int sel_stride, int32_t *sel_lens,
                            int32_t *sel_pages, void *workspace, size_t workspace_bytes,
                            cudaStream_t stream);

/* Workspace of gqa_paged_sparse_decode(): the decode's for B*Hk sequences of one kv head
 * and g = Hq/Hk heads, then the chosen-page lengths and table, then the page scores. */
size_t gqa_paged_sparse_decode_workspace_size(int B, int Hq, int Hk, int head_dim,
                                              int page_size, int pt_stride, int topk, int window,
                                              int num_splits);

/*
 * Sparse decode: the selection, then the decode over the chosen pages, on `stream`.
 * q, pools, page_table, seq_lens, scale, num_splits, out, lse as for gqa_paged_decode()
 * (bf16 pools), except that num_splits = 0 runs the balanced schedule for the decode of the
 * chosen pages (measured faster on the 70B shape than the split count the decode table
 * gives for that size); kt as for gqa_paged_kt_build(); B * Hk <= 65535.  The workspace holds the
 * chosen-page table between the two kernels; zero it once before first use.
 */
int gqa_paged_sparse_decode(const void *q, const void *k_pages, const void *v_pages,
                            const void *kt, const int32_t *page_table, int pt_stride,
                            const int32_t *seq_lens, int B, int Hq, int Hk, int head_dim,
                            int page_size, int num_pages, float scale, int topk, int window,
                            int num_splits, void *out, float *lse, void *workspace,
                            size_t workspace_bytes, cudaStream_t stream);

/*
 * Synchronises `stream`, returns the device error word held in `workspace`
 * (GQA_OK or a negative gqa_status_t) and resets it to GQA_OK.
 */
int gqa_get_error(void *workspace, cudaStream_t stream);

/* Human-readable name of a gqa_status_t value (static string). */
const char *gqa_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* GQA_PAGED_H_ */
