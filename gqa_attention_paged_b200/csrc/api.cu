// api.cu -- the C ABI of libgqa_paged.so (declared in include/gqa_paged.h): argument
// validation, workspace layout, TMA tensor-map encoding and kernel dispatch.  No device
// memory is allocated here; every buffer is the caller's.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "gqa_internal.h"
#include "gqa_paged.h"

using namespace gqa;

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

bool aligned(const void *p, size_t n) { return (reinterpret_cast<uintptr_t>(p) % n) == 0; }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// 2-D view [rows][D] of a KV pool, box = (128 bytes of a row) x box_rows rows, 128B swizzle.
int encode_kv_map(CUtensorMap *map, const void *pages, int kv_dtype, int D, int64_t rows,
                  int box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return GQA_ERR_LAUNCH;
    const int elt = kv_dtype == GQA_KV_FP8_E4M3 ? 1 : 2;
    cuuint64_t gdim[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    cuuint64_t gstride[1] = {(cuuint64_t)D * elt};
    cuuint32_t box[2] = {(cuuint32_t)(128 / elt), (cuuint32_t)box_rows};
    cuuint32_t estride[2] = {1, 1};
    CUresult r = enc(map,
                     elt == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                     const_cast<void *>(pages), gdim, gstride, box, estride,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? GQA_OK : GQA_ERR_LAUNCH;
}

// 3-D view [total_q][Hq][D] of q (or out), box = 64 dims x g heads x T tokens, 128B swizzle.
int encode_q_map(CUtensorMap *map, const void *q, int total_q, int Hq, int D, int g, int T) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return GQA_ERR_LAUNCH;
    cuuint64_t gdim[3] = {(cuuint64_t)D, (cuuint64_t)Hq, (cuuint64_t)total_q};
    cuuint64_t gstride[2] = {(cuuint64_t)D * 2, (cuuint64_t)Hq * D * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)g, (cuuint32_t)T};
    cuuint32_t estride[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(q), gdim, gstride,
                     box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? GQA_OK : GQA_ERR_LAUNCH;
}

bool valid_page_size(int P) { return P == 16 || P == 32 || P == 64; }

int sm_count();

// Split counts measured on one B200 (148 SMs) with `bench.py --sweep splits` (its summary is
// committed under profiles/): Hq=32, Hk=8, head_dim 128, page 16, every sequence the same
// length; rows: units B*Hk (kTabUnitsAt), columns: context in tokens (kTabCtxAt); [0] bf16
// KV, [1] e4m3 KV.  Cells with B * context above 2M tokens were not measured and repeat
// their measured neighbour.
//   kBestSplits: the split schedule's fastest split count (gqa_pick_splits).
//   kAutoSplits: what num_splits = 0 runs: 0 = the balanced schedule, else that split
//     count, where the split schedule measured at least 5% faster than the balanced one
//     (a few short sequences).
constexpr int kTabUnits = 8, kTabCtx = 5;
const int kTabUnitsAt[kTabUnits] = {8, 16, 32, 64, 128, 512, 2048, 8192};
const int kTabCtxAt[kTabCtx] = {512, 2048, 4096, 8192, 32768};
const unsigned char kBestSplits[2][kTabUnits][kTabCtx] = {
    {{8, 16, 16, 32, 32}, {8, 16, 16, 16, 16}, {4, 8, 8, 8, 32}, {4, 4, 4, 16, 32}, {2, 2, 8, 16, 16}, {2, 4, 4, 4, 4}, {1, 1, 1, 1, 1}, {1, 1, 1, 1, 1}},
    {{8, 16, 16, 16, 32}, {8, 8, 16, 16, 16}, {4, 8, 8, 8, 32}, {4, 4, 4, 16, 32}, {2, 2, 8, 16, 16}, {1, 4, 4, 4, 16}, {1, 1, 1, 4, 4}, {1, 1, 1, 1, 1}}};
const unsigned char kAutoSplits[2][kTabUnits][kTabCtx] = {
    {{8, 16, 0, 0, 0}, {8, 0, 0, 16, 0}, {4, 8, 8, 0, 0}, {4, 4, 0, 0, 0}, {2, 0, 0, 0, 0}, {0, 0, 0, 0, 0}, {0, 0, 0, 0, 0}, {0, 0, 0, 0, 0}},
    {{8, 16, 0, 0, 0}, {8, 8, 16, 0, 0}, {4, 8, 8, 0, 0}, {4, 4, 0, 0, 0}, {2, 0, 0, 0, 0}, {0, 0, 0, 0, 0}, {0, 0, 0, 0, 0}, {0, 0, 0, 0, 0}}};

// Index of the entry of `at` nearest to x in log scale.
int nearest_log(const int *at, int n, double x) {
    int best = 0;
    double bd = 1e30;
    const double lx = log(x > 1.0 ? x : 1.0);
    for (int i = 0; i < n; ++i) {
        const double d = fabs(log((double)at[i]) - lx);
        if (d < bd) {
            bd = d;
            best = i;
        }
    }
    return best;
}

// Table cell of (units, context); units are first scaled to 148 SMs.
void split_cell(int B, int Hk, int max_seq_len, int &ui, int &ci) {
    const double units = (double)B * Hk * 148.0 / (double)sm_count();
    ui = nearest_log(kTabUnitsAt, kTabUnits, units);
    ci = nearest_log(kTabCtxAt, kTabCtx, (double)max_seq_len);
}

int clamp_splits(int s, int max_seq_len, int P) {
    const int pages = (max_seq_len + P - 1) / P;
    if (s > pages) s = pages;
    if (s > GQA_MAX_SPLITS) s = GQA_MAX_SPLITS;
    return s < 1 ? 1 : s;
}

// The schedule a decode call runs: 0 = balanced persistent, else the split schedule with
// that many splits.
int decode_schedule(int num_splits, int B, int Hk, int max_seq_len, int P, int kv_dtype) {
    if (num_splits > 0) return num_splits;
    if (B > kStreamMaxBatch) return gqa_pick_splits(B, Hk, max_seq_len, P, kv_dtype);
    if (num_splits == GQA_SPLITS_BALANCED || B <= 0 || Hk <= 0 || P <= 0) return 0;
    int ui, ci;
    split_cell(B, Hk, max_seq_len, ui, ci);
    const int s = kAutoSplits[kv_dtype == GQA_KV_FP8_E4M3 ? 1 : 0][ui][ci];
    return s == 0 ? 0 : clamp_splits(s, max_seq_len, P);
}

// Merge-piece slots of the balanced schedule: 2 per worker, for the largest grid.
size_t stream_k_piece_bytes(int Hq, int Hk, int D) {
    const int g = Hq / Hk;
    const int hpc = g < 16 ? g : 16;
    const size_t slots = (size_t)kStreamMaxSms * kStreamCtasPerSm * kStreamWorkersPerCta * 2;
    const size_t slot_floats = ((size_t)hpc * (D + 1) + 3) / 4 * 4;  // 16-byte aligned slots
    return align_up(slots * slot_floats * sizeof(float), 256);
}


// CTAs of the balanced decode schedule: kStreamCtasPerSm per SM.
int decode_grid() {
    int sms = sm_count();
    if (sms > kStreamMaxSms) sms = kStreamMaxSms;
    return sms * kStreamCtasPerSm;
}

int sm_count() {
    static int cached[256] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 256) return 148;
    if (cached[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
            n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

}  // namespace

namespace gqa {

int decode_check_args(const void *q, const void *k_pages, const void *v_pages,
                      const float *k_scale, const float *v_scale, int kv_dtype,
                      const int32_t *page_table, int pt_stride, const int32_t *seq_lens, int B,
                      int Hq, int Hk, int head_dim, int page_size, int num_pages, int num_splits,
                      const void *out, const float *lse) {
    if (!q || !k_pages || !v_pages || !page_table || !seq_lens || !out) return GQA_ERR_NULL;
    if (kv_dtype != GQA_KV_BF16 && kv_dtype != GQA_KV_FP8_E4M3) return GQA_ERR_DTYPE;
    if (kv_dtype == GQA_KV_FP8_E4M3 && (!k_scale || !v_scale || head_dim != 128))
        return GQA_ERR_DTYPE;
    if (B < 0 || B > 65535 || Hq <= 0 || Hk <= 0 || Hq % Hk != 0 || Hk > 65535 ||
        (head_dim != 64 && head_dim != 128) || !valid_page_size(page_size) || num_pages <= 0 ||
        pt_stride <= 0 || (int64_t)num_pages * Hk * page_size > INT32_MAX ||
        (int64_t)pt_stride * page_size > INT32_MAX)
        return GQA_ERR_SHAPE;
    if (num_splits < GQA_SPLITS_BALANCED || num_splits > GQA_MAX_SPLITS) return GQA_ERR_SPLITS;
    if (!aligned(q, 16) || !aligned(k_pages, 16) || !aligned(v_pages, 16) || !aligned(out, 16) ||
        !aligned(page_table, 4) || !aligned(seq_lens, 4) || (lse && !aligned(lse, 4)))
        return GQA_ERR_ALIGN;
    return GQA_OK;
}

// gqa_paged_decode() and gqa_paged_decode_partial(): out is bf16, or fp32 when out_f32.
int decode_call(const void *q, const void *k_pages, const void *v_pages, const float *k_scale,
                const float *v_scale, int kv_dtype, const int32_t *page_table, int pt_stride,
                const int32_t *seq_lens, int B, int Hq, int Hk, int head_dim, int page_size,
                int num_pages, float scale, int num_splits, int pack_gqa, void *out, int out_f32,
                float *lse, void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    const int chk = decode_check_args(q, k_pages, v_pages, k_scale, v_scale, kv_dtype, page_table,
                                      pt_stride, seq_lens, B, Hq, Hk, head_dim, page_size,
                                      num_pages, num_splits, out, lse);
    if (chk != GQA_OK) return chk;
    if (!workspace) return GQA_ERR_NULL;
    const int sched = decode_schedule(num_splits, B, Hk, pt_stride * page_size, page_size, kv_dtype);
    const bool sk = sched == 0;
    const int S = sk ? 1 : sched;
    const size_t need = gqa_paged_decode_workspace_size(B, Hq, Hk, head_dim, page_size,
                                                        pt_stride * page_size, kv_dtype,
                                                        num_splits);
    if (!aligned(workspace, 256) || workspace_bytes < need) return GQA_ERR_WORKSPACE;
    if (B == 0) return GQA_OK;

    const int64_t rows = (int64_t)num_pages * Hk * page_size;
    CUtensorMap kmap, vmap;
    const int box_rows = decode_tile_tokens(kv_dtype, page_size);
    if (encode_kv_map(&kmap, k_pages, kv_dtype, head_dim, rows, box_rows) != GQA_OK ||
        encode_kv_map(&vmap, v_pages, kv_dtype, head_dim, rows, box_rows) != GQA_OK)
        return GQA_ERR_LAUNCH;

    uint8_t *ws = static_cast<uint8_t *>(workspace);
    DecodeArgs a;
    a.q = q;
    a.k_scale = k_scale;
    a.v_scale = v_scale;
    a.page_table = page_table;
    a.pt_stride = pt_stride;
    a.seq_lens = seq_lens;
    a.B = B;
    a.Hq = Hq;
    a.Hk = Hk;
    a.D = head_dim;
    a.P = page_size;
    a.num_pages = num_pages;
    a.kv_dtype = kv_dtype;
    a.scale = scale;
    a.num_splits = S;
    a.pack_gqa = pack_gqa ? 1 : 0;
    a.out = out;
    a.out_f32 = out_f32;
    a.lse = lse;
    a.err = reinterpret_cast<int *>(ws);
    const size_t rows_q = (size_t)B * Hq;
    a.o_part = S > 1 ? reinterpret_cast<float *>(ws + kWorkspaceHeader) : nullptr;
    a.lse_part = S > 1 ? reinterpret_cast<float *>(
                             ws + kWorkspaceHeader +
                             align_up((size_t)S * rows_q * head_dim * sizeof(float), 256))
                       : nullptr;
    a.stream_k = sk ? 1 : 0;
    a.counters = sk ? reinterpret_cast<int *>(ws + kWorkspaceHeader) : nullptr;
    a.pieces = sk ? reinterpret_cast<float *>(ws + decode_zero_prefix_bytes(B, Hq)) : nullptr;
    a.grid = decode_grid();
    if (launch_decode(a, kmap, vmap, stream) != cudaSuccess) return GQA_ERR_LAUNCH;
    if (S > 1 && launch_lse_combine(a.o_part, a.lse_part, S, (int)rows_q, head_dim, out, lse,
                                    stream, out_f32) != cudaSuccess)
        return GQA_ERR_LAUNCH;
    return GQA_OK;
}

}  // namespace gqa

extern "C" {

const char *gqa_status_string(int s) {
    switch (s) {
        case GQA_OK: return "ok";
        case GQA_ERR_NULL: return "a required pointer is NULL";
        case GQA_ERR_SHAPE: return "unsupported or inconsistent sizes";
        case GQA_ERR_DTYPE: return "unsupported kv dtype / missing fp8 scales";
        case GQA_ERR_SPLITS: return "num_splits out of range";
        case GQA_ERR_WORKSPACE: return "workspace missing, too small or misaligned";
        case GQA_ERR_LAUNCH: return "CUDA launch or driver call failed";
        case GQA_ERR_BAD_PAGE: return "page-table entry or sequence length out of range";
        case GQA_ERR_TIMEOUT: return "a bounded device wait ran out";
        case GQA_ERR_ALIGN: return "pointer not 16-byte aligned";
        default: return "unknown status";
    }
}

int gqa_pick_splits(int B, int Hk, int max_seq_len, int page_size, int kv_dtype) {
    if (B <= 0 || Hk <= 0 || page_size <= 0 || max_seq_len <= 0) return 1;
    int ui, ci;
    split_cell(B, Hk, max_seq_len, ui, ci);
    return clamp_splits(kBestSplits[kv_dtype == GQA_KV_FP8_E4M3 ? 1 : 0][ui][ci], max_seq_len,
                        page_size);
}

size_t gqa_paged_decode_workspace_size(int B, int Hq, int Hk, int head_dim, int page_size,
                                       int max_seq_len, int kv_dtype, int num_splits) {
    const int S = decode_schedule(num_splits, B, Hk, max_seq_len, page_size, kv_dtype);
    if (S == 0 && Hq > 0 && Hk > 0 && Hq % Hk == 0)
        return decode_zero_prefix_bytes(B, Hq) + stream_k_piece_bytes(Hq, Hk, head_dim);
    size_t bytes = kWorkspaceHeader;
    if (S > 1) {
        const size_t rows = (size_t)B * Hq;
        bytes += align_up((size_t)S * rows * head_dim * sizeof(float), 256);
        bytes += align_up((size_t)S * rows * sizeof(float), 256);
    }
    return bytes;
}

int gqa_paged_decode_kernel_launches(int B, int Hq, int Hk, int head_dim, int page_size,
                                     int max_seq_len, int kv_dtype, int num_splits,
                                     int pack_gqa) {
    (void)head_dim;
    if (B <= 0 || Hq <= 0 || Hk <= 0 || Hq % Hk != 0 || page_size <= 0) return 0;
    const int S = decode_schedule(num_splits, B, Hk, max_seq_len, page_size, kv_dtype);
    if (S == 0) return decode_defers_merge(B, Hq, Hk, pack_gqa ? 1 : 0, decode_grid()) ? 2 : 1;
    return S > 1 ? 2 : 1;
}

size_t gqa_paged_prefill_workspace_size(int total_q, int Hq, int head_dim) {
    (void)Hq;
    (void)head_dim;
    return prefill_workspace_bytes(total_q < 0 ? 0 : total_q);
}

int gqa_paged_decode(const void *q, const void *k_pages, const void *v_pages,
                     const float *k_scale, const float *v_scale, int kv_dtype,
                     const int32_t *page_table, int pt_stride, const int32_t *seq_lens, int B,
                     int Hq, int Hk, int head_dim, int page_size, int num_pages, float scale,
                     int num_splits, int pack_gqa, void *out, float *lse, void *workspace,
                     size_t workspace_bytes, cudaStream_t stream) {
    return decode_call(q, k_pages, v_pages, k_scale, v_scale, kv_dtype, page_table, pt_stride,
                       seq_lens, B, Hq, Hk, head_dim, page_size, num_pages, scale, num_splits,
                       pack_gqa, out, 0, lse, workspace, workspace_bytes, stream);
}

int gqa_paged_decode_partial(const void *q, const void *k_pages, const void *v_pages,
                             const float *k_scale, const float *v_scale, int kv_dtype,
                             const int32_t *page_table, int pt_stride, const int32_t *seq_lens,
                             int B, int Hq, int Hk, int head_dim, int page_size, int num_pages,
                             float scale, int num_splits, int pack_gqa, float *o_part,
                             float *lse_part, void *workspace, size_t workspace_bytes,
                             cudaStream_t stream) {
    if (!lse_part) return GQA_ERR_NULL;
    return decode_call(q, k_pages, v_pages, k_scale, v_scale, kv_dtype, page_table, pt_stride,
                       seq_lens, B, Hq, Hk, head_dim, page_size, num_pages, scale, num_splits,
                       pack_gqa, o_part, 1, lse_part, workspace, workspace_bytes, stream);
}

int gqa_paged_prefill(const void *q, const int32_t *cu_q, const void *k_pages,
                      const void *v_pages, const int32_t *page_table, int pt_stride,
                      const int32_t *seq_lens, int B, int Hq, int Hk, int head_dim,
                      int page_size, int num_pages, float scale, int causal, int total_q,
                      int max_q_len, void *out, float *lse, void *workspace,
                      size_t workspace_bytes, cudaStream_t stream) {
    if (!q || !cu_q || !k_pages || !v_pages || !page_table || !seq_lens || !out || !workspace)
        return GQA_ERR_NULL;
    if (B < 0 || B > 65535 || Hq <= 0 || Hk <= 0 || Hq % Hk != 0 || Hk > 65535 ||
        Hq / Hk > 128 || (head_dim != 64 && head_dim != 128) || !valid_page_size(page_size) || num_pages <= 0 ||
        pt_stride <= 0 || total_q < 0 || max_q_len < 0 || !(scale > 0.f) ||
        (int64_t)num_pages * Hk * page_size > INT32_MAX ||
        (int64_t)pt_stride * page_size > INT32_MAX)
        return GQA_ERR_SHAPE;
    if (!aligned(q, 16) || !aligned(k_pages, 16) || !aligned(v_pages, 16) || !aligned(out, 16) ||
        !aligned(page_table, 4) || !aligned(seq_lens, 4) || !aligned(cu_q, 4) ||
        (lse && !aligned(lse, 4)))
        return GQA_ERR_ALIGN;
    if (!aligned(workspace, 256) ||
        workspace_bytes < gqa_paged_prefill_workspace_size(total_q, Hq, head_dim))
        return GQA_ERR_WORKSPACE;
    if (B == 0 || total_q == 0 || max_q_len == 0) return GQA_OK;
    const int g = Hq / Hk;
    const int T = 128 / g;
    // work items (pairs of query tiles) per sequence, and the launch's upper bound on them
    const int64_t items_per_seq = ((int64_t)max_q_len + 2 * T - 1) / (2 * T);
    if (items_per_seq > 65535 || (int64_t)B * items_per_seq * Hk > INT32_MAX) return GQA_ERR_SHAPE;
    const int64_t rows = (int64_t)num_pages * Hk * page_size;
    CUtensorMap kmap, vmap, qmap;
    if (encode_kv_map(&kmap, k_pages, GQA_KV_BF16, head_dim, rows, 16) != GQA_OK ||
        encode_kv_map(&vmap, v_pages, GQA_KV_BF16, head_dim, rows, 16) != GQA_OK ||
        encode_q_map(&qmap, q, total_q, Hq, head_dim, g, T) != GQA_OK)
        return GQA_ERR_LAUNCH;
    PrefillArgs a;
    a.q = q;
    a.cu_q = cu_q;
    a.page_table = page_table;
    a.pt_stride = pt_stride;
    a.seq_lens = seq_lens;
    a.B = B;
    a.Hq = Hq;
    a.Hk = Hk;
    a.D = head_dim;
    a.P = page_size;
    a.num_pages = num_pages;
    a.scale = scale;
    a.causal = causal ? 1 : 0;
    a.total_q = total_q;
    a.max_q_len = max_q_len;
    a.out = out;
    a.lse = lse;
    a.err = reinterpret_cast<int *>(workspace);
    a.plan = reinterpret_cast<int *>(static_cast<uint8_t *>(workspace) + kWorkspaceHeader);
    return launch_prefill(a, kmap, vmap, qmap, stream) == cudaSuccess ? GQA_OK : GQA_ERR_LAUNCH;
}

int lse_combine(const float *o_part, const float *lse_part, int num_splits, int rows,
                int head_dim, void *out, float *lse, cudaStream_t stream) {
    if (!o_part || !lse_part || !out) return GQA_ERR_NULL;
    if (rows < 0 || (head_dim != 64 && head_dim != 128)) return GQA_ERR_SHAPE;
    if (num_splits < 1 || num_splits > GQA_MAX_SPLITS) return GQA_ERR_SPLITS;
    if (!aligned(o_part, 16) || !aligned(out, 16) || !aligned(lse_part, 4) ||
        (lse && !aligned(lse, 4)))
        return GQA_ERR_ALIGN;
    return launch_lse_combine(o_part, lse_part, num_splits, rows, head_dim, out, lse, stream) ==
                   cudaSuccess
               ? GQA_OK
               : GQA_ERR_LAUNCH;
}

int gqa_paged_gather(const void *k_pages, const void *v_pages, const int32_t *page_table,
                     int pt_stride, const int32_t *seq_lens, const int64_t *cu_kv, int B,
                     int Hk, int head_dim, int page_size, int num_pages, int elem_bytes,
                     void *k_out, void *v_out, cudaStream_t stream) {
    if (!k_pages || !v_pages || !page_table || !seq_lens || !cu_kv || !k_out || !v_out)
        return GQA_ERR_NULL;
    if (B < 0 || B > 65535 || Hk <= 0 || (head_dim != 64 && head_dim != 128) ||
        !valid_page_size(page_size) || num_pages <= 0 || pt_stride <= 0 ||
        (elem_bytes != 1 && elem_bytes != 2))
        return GQA_ERR_SHAPE;
    if (!aligned(k_pages, 16) || !aligned(v_pages, 16) || !aligned(k_out, 16) ||
        !aligned(v_out, 16) || !aligned(cu_kv, 8))
        return GQA_ERR_ALIGN;
    if (B == 0) return GQA_OK;
    return launch_gather(k_pages, v_pages, page_table, pt_stride, seq_lens, cu_kv, B, Hk,
                         head_dim, page_size, num_pages, elem_bytes, k_out, v_out, stream) ==
                   cudaSuccess
               ? GQA_OK
               : GQA_ERR_LAUNCH;
}

int gqa_paged_append_kv(const void *k_new, const void *v_new, void *k_pages, void *v_pages,
                        float *k_scale, float *v_scale, int kv_dtype, const int32_t *page_table,
                        int pt_stride, const int32_t *seq_lens, int B, int Hk, int head_dim,
                        int page_size, int num_pages, void *workspace, cudaStream_t stream) {
    if (!k_new || !v_new || !k_pages || !v_pages || !page_table || !seq_lens || !workspace)
        return GQA_ERR_NULL;
    if (kv_dtype != GQA_KV_BF16 && kv_dtype != GQA_KV_FP8_E4M3) return GQA_ERR_DTYPE;
    if (kv_dtype == GQA_KV_FP8_E4M3 && (!k_scale || !v_scale)) return GQA_ERR_DTYPE;
    if (B < 0 || B > 65535 || Hk <= 0 || Hk > 65535 || (head_dim != 64 && head_dim != 128) ||
        !valid_page_size(page_size) || num_pages <= 0 || pt_stride <= 0 ||
        (int64_t)num_pages * Hk * page_size > INT32_MAX ||
        (int64_t)pt_stride * page_size > INT32_MAX)
        return GQA_ERR_SHAPE;
    if (!aligned(k_new, 2) || !aligned(v_new, 2) || !aligned(k_pages, 2) ||
        !aligned(v_pages, 2) || !aligned(page_table, 4) || !aligned(seq_lens, 4) ||
        !aligned(workspace, 256) || (k_scale && !aligned(k_scale, 4)) ||
        (v_scale && !aligned(v_scale, 4)))
        return GQA_ERR_ALIGN;
    AppendArgs a;
    a.k_new = k_new;
    a.v_new = v_new;
    a.k_pages = k_pages;
    a.v_pages = v_pages;
    a.k_scale = k_scale;
    a.v_scale = v_scale;
    a.kv_dtype = kv_dtype;
    a.page_table = page_table;
    a.pt_stride = pt_stride;
    a.seq_lens = seq_lens;
    a.B = B;
    a.Hk = Hk;
    a.D = head_dim;
    a.P = page_size;
    a.num_pages = num_pages;
    a.err = reinterpret_cast<int *>(workspace);
    return launch_append(a, stream) == cudaSuccess ? GQA_OK : GQA_ERR_LAUNCH;
}

int gqa_paged_append_decode(const void *q, const void *k_new, const void *v_new, void *k_pages,
                            void *v_pages, float *k_scale, float *v_scale, int kv_dtype,
                            const int32_t *page_table, int pt_stride, const int32_t *seq_lens,
                            int B, int Hq, int Hk, int head_dim, int page_size, int num_pages,
                            float scale, int num_splits, int pack_gqa, void *out, float *lse,
                            void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    // the decode's checks first, so that a call it would reject changes nothing
    if (!q || !out) return GQA_ERR_NULL;
    if (Hq <= 0 || Hk <= 0 || Hq % Hk != 0) return GQA_ERR_SHAPE;
    if (num_splits < GQA_SPLITS_BALANCED || num_splits > GQA_MAX_SPLITS) return GQA_ERR_SPLITS;
    if (kv_dtype == GQA_KV_FP8_E4M3 && head_dim != 128) return GQA_ERR_DTYPE;
    if (!workspace || !aligned(workspace, 256)) return workspace ? GQA_ERR_WORKSPACE : GQA_ERR_NULL;
    if (!aligned(q, 16) || !aligned(k_pages, 16) || !aligned(v_pages, 16) || !aligned(out, 16) ||
        (lse && !aligned(lse, 4)))
        return GQA_ERR_ALIGN;
    if (workspace_bytes < gqa_paged_decode_workspace_size(B, Hq, Hk, head_dim, page_size,
                                                          pt_stride * page_size, kv_dtype,
                                                          num_splits))
        return GQA_ERR_WORKSPACE;
    const int r = gqa_paged_append_kv(k_new, v_new, k_pages, v_pages, k_scale, v_scale,
                                      kv_dtype, page_table, pt_stride, seq_lens, B, Hk,
                                      head_dim, page_size, num_pages, workspace, stream);
    if (r != GQA_OK) return r;
    return gqa_paged_decode(q, k_pages, v_pages, k_scale, v_scale, kv_dtype, page_table,
                            pt_stride, seq_lens, B, Hq, Hk, head_dim, page_size, num_pages,
                            scale, num_splits, pack_gqa, out, lse, workspace, workspace_bytes,
                            stream);
}

int gqa_paged_kt_build(const void *k_pages, const int32_t *page_table, int pt_stride,
                       const int32_t *seq_lens, int B, int Hk, int head_dim, int page_size,
                       int num_pages, void *kt, void *workspace, cudaStream_t stream) {
    if (!k_pages || !page_table || !seq_lens || !kt || !workspace) return GQA_ERR_NULL;
    if (B < 0 || B > 65535 || Hk <= 0 || (head_dim != 64 && head_dim != 128) ||
        !valid_page_size(page_size) || num_pages <= 0 || pt_stride <= 0 ||
        (int64_t)num_pages * Hk * page_size > INT32_MAX || (int64_t)pt_stride * page_size > INT32_MAX)
        return GQA_ERR_SHAPE;
    if (!aligned(k_pages, 16) || !aligned(kt, 16) || !aligned(page_table, 4) ||
        !aligned(seq_lens, 4) || !aligned(workspace, 256))
        return GQA_ERR_ALIGN;
    return launch_kt_build(k_pages, page_table, pt_stride, seq_lens, B, Hk, head_dim, page_size,
                           num_pages, kt, static_cast<int *>(workspace), stream) == cudaSuccess
               ? GQA_OK
               : GQA_ERR_LAUNCH;
}

int gqa_paged_kt_append(const void *k_new, const int32_t *page_table, int pt_stride,
                        const int32_t *seq_lens, int B, int Hk, int head_dim, int page_size,
                        int num_pages, void *kt, void *workspace, cudaStream_t stream) {
    if (!k_new || !page_table || !seq_lens || !kt || !workspace) return GQA_ERR_NULL;
    if (B < 0 || B > 65535 || Hk <= 0 || (head_dim != 64 && head_dim != 128) ||
        !valid_page_size(page_size) || num_pages <= 0 || pt_stride <= 0 ||
        (int64_t)num_pages * Hk * page_size > INT32_MAX || (int64_t)pt_stride * page_size > INT32_MAX)
        return GQA_ERR_SHAPE;
    if (!aligned(k_new, 2) || !aligned(kt, 16) || !aligned(page_table, 4) ||
        !aligned(seq_lens, 4) || !aligned(workspace, 256))
        return GQA_ERR_ALIGN;
    return launch_kt_append(k_new, page_table, pt_stride, seq_lens, B, Hk, head_dim, page_size,
                            num_pages, kt, static_cast<int *>(workspace), stream) == cudaSuccess
               ? GQA_OK
               : GQA_ERR_LAUNCH;
}

int gqa_paged_sparse_table_stride(int pt_stride, int page_size, int topk, int window) {
    if (pt_stride <= 0 || page_size <= 0 || topk < 0 || window < 0) return 0;
    // topk earlier pages plus the pages a window of `window` tokens can touch
    const int64_t win_pages = window > 0 ? ((int64_t)window + page_size - 1) / page_size + 1 : 0;
    const int64_t s = (int64_t)topk + win_pages;
    return (int)(s < pt_stride ? s : pt_stride);
}

size_t gqa_paged_sparse_select_workspace_size(int B, int Hk, int pt_stride) {
    if (B < 0 || Hk <= 0 || pt_stride <= 0) return 0;
    return kWorkspaceHeader + align_up((size_t)B * Hk * pt_stride * sizeof(uint32_t), 256);
}

int gqa_paged_sparse_select(const void *q, const void *kt, const int32_t *page_table,
                            int pt_stride, const int32_t *seq_lens, int B, int Hq, int Hk,
                            int head_dim, int page_size, int num_pages, int topk, int window,
                            int32_t *sel_table, int sel_stride, int32_t *sel_lens,
                            int32_t *sel_pages, void *workspace, size_t workspace_bytes,
                            cudaStream_t stream) {
    if (!q || !kt || !page_table || !seq_lens || !sel_table || !sel_lens || !workspace)
        return GQA_ERR_NULL;
    if (B < 0 || B > 65535 || Hq <= 0 || Hk <= 0 || Hq % Hk != 0 ||
        Hq / Hk > kSparseMaxGroup || (head_dim != 64 && head_dim != 128) ||
        !valid_page_size(page_size) || num_pages <= 0 || pt_stride <= 0 ||
        pt_stride > kSparseMaxPages || topk < 0 || window < 0 ||
        sel_stride < gqa_paged_sparse_table_stride(pt_stride, page_size, topk, window) ||
        (int64_t)num_pages * Hk * page_size > INT32_MAX)
        return GQA_ERR_SHAPE;
    if (!aligned(q, 16) || !aligned(kt, 16) || !aligned(page_table, 4) || !aligned(seq_lens, 4) ||
        !aligned(sel_table, 4) || !aligned(sel_lens, 4) || (sel_pages && !aligned(sel_pages, 4)))
        return GQA_ERR_ALIGN;
    if (!aligned(workspace, 256) ||
        workspace_bytes < gqa_paged_sparse_select_workspace_size(B, Hk, pt_stride))
        return GQA_ERR_WORKSPACE;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    return launch_sparse_select(q, kt, page_table, pt_stride, seq_lens, B, Hq, Hk, head_dim,
                                page_size, num_pages, topk, window, sel_table, sel_stride,
                                sel_lens, sel_pages, reinterpret_cast<uint32_t *>(ws + kWorkspaceHeader),
                                reinterpret_cast<int *>(ws), stream) == cudaSuccess
               ? GQA_OK
               : GQA_ERR_LAUNCH;
}

// The schedule of the decode over the chosen pages: num_splits = 0 runs the balanced
// schedule.  The dense table's pick for that size (8 splits for 32 one-kv-head sequences of
// ~2K tokens) measured slower on the 70B shape (Hq/Hk = 8, top 32 pages + window):
// 32.7 against 31.0 us per sparse step.
int sparse_decode_splits(int num_splits) { return num_splits == 0 ? GQA_SPLITS_BALANCED : num_splits; }

size_t gqa_paged_sparse_decode_workspace_size(int B, int Hq, int Hk, int head_dim,
                                              int page_size, int pt_stride, int topk, int window,
                                              int num_splits) {
    if (B < 0 || Hq <= 0 || Hk <= 0 || Hq % Hk != 0) return 0;
    const int ss = gqa_paged_sparse_table_stride(pt_stride, page_size, topk, window);
    if (ss <= 0) return 0;
    const int Bv = B * Hk;
    return gqa_paged_decode_workspace_size(Bv, Hq / Hk, 1, head_dim, page_size, ss * page_size,
                                           GQA_KV_BF16, sparse_decode_splits(num_splits)) +
           align_up((size_t)Bv * sizeof(int32_t), 256) +
           align_up((size_t)Bv * ss * sizeof(int32_t), 256) +
           align_up((size_t)Bv * pt_stride * sizeof(uint32_t), 256);
}

int gqa_paged_sparse_decode(const void *q, const void *k_pages, const void *v_pages,
                            const void *kt, const int32_t *page_table, int pt_stride,
                            const int32_t *seq_lens, int B, int Hq, int Hk, int head_dim,
                            int page_size, int num_pages, float scale, int topk, int window,
                            int num_splits, void *out, float *lse, void *workspace,
                            size_t workspace_bytes, cudaStream_t stream) {
    if (!q || !k_pages || !v_pages || !kt || !page_table || !seq_lens || !out || !workspace)
        return GQA_ERR_NULL;
    if (B < 0 || B > 65535 || Hq <= 0 || Hk <= 0 || Hq % Hk != 0 ||
        Hq / Hk > kSparseMaxGroup || (head_dim != 64 && head_dim != 128) ||
        !valid_page_size(page_size) || num_pages <= 0 || pt_stride <= 0 ||
        pt_stride > kSparseMaxPages || topk < 0 || window < 0 ||
        (int64_t)B * Hk > 65535 || (int64_t)num_pages * Hk * page_size > INT32_MAX ||
        (int64_t)pt_stride * page_size > INT32_MAX)
        return GQA_ERR_SHAPE;
    if (num_splits < 0 || num_splits > GQA_MAX_SPLITS) return GQA_ERR_SPLITS;
    if (!aligned(q, 16) || !aligned(k_pages, 16) || !aligned(v_pages, 16) || !aligned(kt, 16) ||
        !aligned(out, 16) || !aligned(page_table, 4) || !aligned(seq_lens, 4) ||
        (lse && !aligned(lse, 4)))
        return GQA_ERR_ALIGN;
    const size_t need = gqa_paged_sparse_decode_workspace_size(B, Hq, Hk, head_dim, page_size,
                                                               pt_stride, topk, window, num_splits);
    if (!aligned(workspace, 256) || workspace_bytes < need) return GQA_ERR_WORKSPACE;
    if (B == 0) return GQA_OK;
    const int ss = gqa_paged_sparse_table_stride(pt_stride, page_size, topk, window);
    const int Bv = B * Hk, g = Hq / Hk;
    const int dsplits = sparse_decode_splits(num_splits);
    const size_t dws = gqa_paged_decode_workspace_size(Bv, g, 1, head_dim, page_size,
                                                       ss * page_size, GQA_KV_BF16, dsplits);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    int32_t *sel_lens = reinterpret_cast<int32_t *>(ws + dws);
    int32_t *sel_table = reinterpret_cast<int32_t *>(ws + dws + align_up((size_t)Bv * 4, 256));
    uint32_t *keys = reinterpret_cast<uint32_t *>(ws + dws + align_up((size_t)Bv * 4, 256) +
                                                  align_up((size_t)Bv * ss * 4, 256));
    if (launch_sparse_select(q, kt, page_table, pt_stride, seq_lens, B, Hq, Hk, head_dim,
                             page_size, num_pages, topk, window, sel_table, ss, sel_lens, nullptr,
                             keys, reinterpret_cast<int *>(ws), stream) != cudaSuccess)
        return GQA_ERR_LAUNCH;
    // the chosen pages of every (sequence, kv head) as one sequence of a decode with one kv
    // head: q [B*Hk][g][D], pools [num_pages*Hk][1][P][D], out [B*Hk][g][D]
    return decode_call(q, k_pages, v_pages, nullptr, nullptr, GQA_KV_BF16, sel_table, ss,
                       sel_lens, Bv, g, 1, head_dim, page_size, num_pages * Hk, scale,
                       dsplits, 1, out, 0, lse, workspace, dws, stream);
}

int gqa_get_error(void *workspace, cudaStream_t stream) {
    if (!workspace) return GQA_ERR_NULL;
    int err = 0;
    if (cudaMemcpyAsync(&err, workspace, sizeof(int), cudaMemcpyDeviceToHost, stream) !=
            cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess)
        return GQA_ERR_LAUNCH;
    if (err != 0) {
        if (cudaMemsetAsync(workspace, 0, sizeof(int), stream) != cudaSuccess ||
            cudaStreamSynchronize(stream) != cudaSuccess)
            return GQA_ERR_LAUNCH;
    }
    return err;
}

}  // extern "C"
