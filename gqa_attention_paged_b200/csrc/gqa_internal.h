// gqa_internal.h -- host-side interfaces between the C-ABI layer (api.cu) and the kernel
// launchers (decode.cu, combine.cu, gather.cu, prefill.cu).  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime_api.h>
#include <stddef.h>
#include <stdint.h>

namespace gqa {

constexpr size_t kWorkspaceHeader = 256;  // bytes before any scratch: holds the error word

struct DecodeArgs {
    const void *q;
    const float *k_scale, *v_scale;
    const int32_t *page_table;
    int pt_stride;
    const int32_t *seq_lens;
    int B, Hq, Hk, D, P, num_pages;
    int kv_dtype;
    float scale;
    int num_splits;
    int pack_gqa;
    void *out;        // bf16 [B][Hq][D], or fp32 when out_f32
    int out_f32;      // 1: write the normalised result in fp32 (gqa_paged_decode_partial)
    float *lse;
    float *o_part, *lse_part;  // scratch for num_splits > 1
    int *err;
    // balanced persistent schedule (num_splits == 0, B <= kStreamMaxBatch)
    int stream_k;
    int *counters;  // [B * units] merge counters of the last-piece merge; zero between launches
    float *pieces;  // [workers * 2][heads per CTA][D + 1]
    int grid;       // persistent CTAs
};

// Largest batch the balanced persistent decode schedule takes (its per-CTA tile prefix
// over sequences lives in shared memory).
constexpr int kStreamMaxBatch = 2048;
// Persistent decode CTAs per SM and the SM count the workspace is sized for.
constexpr int kStreamCtasPerSm = 2;
constexpr int kStreamMaxSms = 160;
constexpr int kStreamWorkersPerCta = 4;

constexpr int kStreamMaxWorkers = kStreamMaxSms * kStreamCtasPerSm * kStreamWorkersPerCta;

// Packed query heads per decode CTA: the whole group with PackGQA (up to 16, the wide
// instance for groups above 8), else one head.
inline int decode_heads_per_cta(int Hq, int Hk, int pack_gqa) {
    const int g = Hq / Hk;
    const int cap = g > 8 ? 16 : 8;
    return pack_gqa ? (g < cap ? g : cap) : 1;
}
// A balanced-schedule launch whose units average more than this many workers each leaves
// its pieces to a second kernel, which merges every cut unit in parallel; otherwise the
// last piece of each unit merges the unit in the same launch, reading the unit's pieces
// one after another.  Measured at ctx 2048: 9 workers per unit (B=16) 32.8 -> 29.8 us
// with the second kernel, 4.6 (B=32) no gain, 2.3 (B=64) 91.9 -> 100.7 us.  The 16-head instance
// (groups above 8) always leaves them: with the merge in the same launch its streaming
// loop spills, and it measured 1.3-1.9x slower at B=64 (Hq/Hk = 32/2 and 64/4) and no
// faster anywhere.
constexpr int kDeferMinWorkersPerUnit = 8;
inline bool decode_defers_merge(int B, int Hq, int Hk, int pack_gqa, int grid) {
    const int g = Hq / Hk, hpc = decode_heads_per_cta(Hq, Hk, pack_gqa);
    if (hpc > 8) return true;
    const long long units = (long long)B * Hk * ((g + hpc - 1) / hpc);
    return (long long)grid * kStreamWorkersPerCta > (long long)kDeferMinWorkersPerUnit * units;
}

// Bytes at the start of a decode workspace that must be zero before a launch: the error
// word header, then the balanced schedule's merge counters, one per (sequence, head).
inline size_t decode_zero_prefix_bytes(int B, int Hq) {
    return kWorkspaceHeader + ((size_t)B * Hq * sizeof(int) + 255) / 256 * 256;
}

// Host-side checks of gqa_paged_decode()'s arguments other than the workspace: GQA_OK or
// the status the call returns (nothing is enqueued by a call that fails them).
int decode_check_args(const void *q, const void *k_pages, const void *v_pages,
                      const float *k_scale, const float *v_scale, int kv_dtype,
                      const int32_t *page_table, int pt_stride, const int32_t *seq_lens, int B,
                      int Hq, int Hk, int head_dim, int page_size, int num_pages, int num_splits,
                      const void *out, const float *lse);

// Launch the decode kernel on `stream` (for launches whose units are cut into many pieces,
// followed by the kernel that merges the pieces).  The tensor maps describe the
// K and V pools as 2-D arrays [num_pages*Hk*P rows][D].
cudaError_t launch_decode(const DecodeArgs &a, const CUtensorMap &kmap, const CUtensorMap &vmap,
                          cudaStream_t stream);

// out is bf16 [rows][D], or fp32 when out_f32.
cudaError_t launch_lse_combine(const float *o_part, const float *lse_part, int num_splits,
                               int rows, int D, void *out, float *lse, cudaStream_t stream,
                               int out_f32 = 0);

cudaError_t launch_gather(const void *k_pages, const void *v_pages, const int32_t *page_table,
                          int pt_stride, const int32_t *seq_lens, const int64_t *cu_kv, int B,
                          int Hk, int D, int P, int num_pages, int elem_bytes, void *k_out,
                          void *v_out, cudaStream_t stream);

struct PrefillArgs {
    const void *q;
    const int32_t *cu_q;
    const int32_t *page_table;
    int pt_stride;
    const int32_t *seq_lens;
    int B, Hq, Hk, D, P, num_pages;
    float scale;
    int causal;
    int total_q, max_q_len;
    void *out;
    float *lse;
    int *err;
    int *plan;  // [1 + items]: count, then (b << 16 | query-tile pair) longest first
};

// Work items of a prefill launch (pairs of query tiles) are ordered longest first by a
// one-CTA plan kernel; costs are binned by KV tiles up to this many.
constexpr int kPlanBins = 4096;
// Bytes of the prefill workspace: the error-word header, then the plan (one int per
// item, at most one item per query token, plus the count).
inline size_t prefill_workspace_bytes(int total_q) {
    return kWorkspaceHeader + ((size_t)(total_q + 1) * sizeof(int) + 255) / 256 * 256;
}

cudaError_t launch_prefill(const PrefillArgs &a, const CUtensorMap &kmap,
                           const CUtensorMap &vmap, const CUtensorMap &qmap,
                           cudaStream_t stream);

// KV append: the new token of each sequence into its page (append.cu).
struct AppendArgs {
    const void *k_new, *v_new;  // bf16 [B][Hk][D]
    void *k_pages, *v_pages;
    float *k_scale, *v_scale;   // e4m3 only
    int kv_dtype;
    const int32_t *page_table;
    int pt_stride;
    const int32_t *seq_lens;
    int B, Hk, D, P, num_pages;
    int *err;
};
cudaError_t launch_append(const AppendArgs &a, cudaStream_t stream);

// Page-level top-K sparse decode (sparse.cu).  KT cache: bf16 [num_pages][Hk][D][2].
cudaError_t launch_kt_build(const void *k_pages, const int32_t *page_table, int pt_stride,
                            const int32_t *seq_lens, int B, int Hk, int D, int P, int num_pages,
                            void *kt, int *err, cudaStream_t stream);
cudaError_t launch_kt_append(const void *k_new, const int32_t *page_table, int pt_stride,
                             const int32_t *seq_lens, int B, int Hk, int D, int P, int num_pages,
                             void *kt, int *err, cudaStream_t stream);
// The scores of the selection go to `keys` [B*Hk][pt_stride] (order-preserving uint32).
cudaError_t launch_sparse_select(const void *q, const void *kt, const int32_t *page_table,
                                 int pt_stride, const int32_t *seq_lens, int B, int Hq, int Hk,
                                 int D, int P, int num_pages, int topk, int window,
                                 int32_t *sel_table, int sel_stride, int32_t *sel_lens,
                                 int32_t *sel_pages, uint32_t *keys, int *err,
                                 cudaStream_t stream);
// Largest page table (pages per sequence) and group the sparse selection takes.
constexpr int kSparseMaxPages = 16384;
constexpr int kSparseMaxGroup = 16;

// Tokens per decode pipeline stage (the TMA box height of the KV tensor maps): 32 for
// e4m3 KV on pages of at least 32 tokens, else 16.
inline int decode_tile_tokens(int kv_dtype, int page_size) {
    return (kv_dtype == 1 && page_size >= 32) ? 32 : 16;
}

}  // namespace gqa
