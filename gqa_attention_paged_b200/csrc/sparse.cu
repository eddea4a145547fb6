// sparse.cu -- page-level top-K sparse decode: the decode stage of RocketKV as
// "TensorRT-LLM 如何用 sparse_attention_config 配置 Sparse Attention 降低长上下文推理开销"
// (RocketKV configuration section) sets it up: an auxiliary KT cache scores every page of
// a sequence, and the decode attends to the `topk` best pages plus the pages holding the
// most recent `window` tokens, skipping the rest.
//
//   KT entry of (page, kv head): element-wise min and max of the page's keys over its
//     valid tokens, bf16 [num_pages][Hk][D][2] (min, max interleaved per dim).
//   Page score for kv head j: sum over its g query heads h of
//     sum_d max(q_hd * min_d, q_hd * max_d)  -- the largest q.k over the box [min, max],
//     an upper bound of q.k for every key of the page; fp32, d ascending per head, then
//     heads ascending.  Every product of two bf16 values is exact in fp32, so the sums
//     round the same way wherever they are computed in this order.
//   Selection per (sequence, kv head): the window pages, plus the `topk` highest-scoring
//     earlier pages (equal scores: the lower logical page first), all earlier pages when
//     there are no more than `topk` of them.
//   Attention: the decode of this library over the chosen pages only.  Each (sequence,
//     kv head) becomes one sequence of a derived decode problem with one kv head: its
//     chosen pages, in ascending logical order, form its page table (entry =
//     physical page * Hk + kv head, a (page, kv head) block of the pool seen as
//     [num_pages * Hk][1][P][D]), so the balanced decode kernel runs unchanged and every
//     chosen KV byte is still read once for all g heads of the group.
#include "gqa_device.cuh"
#include "gqa_internal.h"

namespace gqa {
namespace {

constexpr int kSelThreads = 512;
constexpr int kSelChunk = 64;  // pages scored per round

// Order-preserving map of an fp32 score to an unsigned key (larger score, larger key).
__device__ __forceinline__ uint32_t score_key(float s) {
    const uint32_t u = __float_as_uint(s);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float bf16_bits_f32(uint32_t bits16) {
    return __uint_as_float(bits16 << 16);
}

// ---------------------------------------------------------------------------- KT build
// One CTA per (logical page, sequence); threads over (kv head, dim pair).
__global__ void __launch_bounds__(256) kt_build_kernel(const uint16_t *__restrict__ k_pages,
                                                       const int32_t *__restrict__ page_table,
                                                       int pt_stride,
                                                       const int32_t *__restrict__ seq_lens,
                                                       int Hk, int D, int P, int num_pages,
                                                       uint16_t *__restrict__ kt, int *err) {
    const int p = blockIdx.x, b = blockIdx.y;
    int L = seq_lens[b];
    if (L < 0 || L > pt_stride * P) {
        if (threadIdx.x == 0 && p == 0) set_error(err, GQA_ERR_BAD_PAGE);
        L = L < 0 ? 0 : pt_stride * P;
    }
    if (p * P >= L) return;
    const int n = min(P, L - p * P);
    const int phys = page_table[(size_t)b * pt_stride + p];
    if (phys < 0 || phys >= num_pages) {
        if (threadIdx.x == 0) set_error(err, GQA_ERR_BAD_PAGE);
        return;
    }
    const int pairs = D / 2;
    for (int e = threadIdx.x; e < Hk * pairs; e += blockDim.x) {
        const int kvh = e / pairs, d = (e % pairs) * 2;
        const uint32_t *src = reinterpret_cast<const uint32_t *>(
            k_pages + (((size_t)phys * Hk + kvh) * P) * D + d);
        float mn0 = INFINITY, mx0 = -INFINITY, mn1 = INFINITY, mx1 = -INFINITY;
#pragma unroll 8
        for (int t = 0; t < n; ++t) {
            const uint32_t w = __ldg(src + (size_t)t * (D / 2));
            const float v0 = bf16_bits_f32(w & 0xffffu), v1 = bf16_bits_f32(w >> 16);
            mn0 = v0 < mn0 ? v0 : mn0;
            mx0 = v0 > mx0 ? v0 : mx0;
            mn1 = v1 < mn1 ? v1 : mn1;
            mx1 = v1 > mx1 ? v1 : mx1;
        }
        // min and max of bf16 values are bf16 values: the top halves are exact
        uint2 o;
        o.x = (__float_as_uint(mn0) >> 16) | (__float_as_uint(mx0) & 0xffff0000u);
        o.y = (__float_as_uint(mn1) >> 16) | (__float_as_uint(mx1) & 0xffff0000u);
        *reinterpret_cast<uint2 *>(kt + (((size_t)phys * Hk + kvh) * D + d) * 2) = o;
    }
}

// ---------------------------------------------------------------------------- KT append
// The new token (position L - 1) of every sequence: a token that opens a page sets the
// page's entry to (k, k); a later one widens it.  One CTA per sequence.
__global__ void __launch_bounds__(256) kt_append_kernel(const uint16_t *__restrict__ k_new,
                                                        const int32_t *__restrict__ page_table,
                                                        int pt_stride,
                                                        const int32_t *__restrict__ seq_lens,
                                                        int Hk, int D, int P, int num_pages,
                                                        uint16_t *__restrict__ kt, int *err) {
    const int b = blockIdx.x;
    const int L = seq_lens[b];
    if (L <= 0) return;
    if (L > pt_stride * P) {
        if (threadIdx.x == 0) set_error(err, GQA_ERR_BAD_PAGE);
        return;
    }
    const int t = L - 1;
    const int phys = page_table[(size_t)b * pt_stride + t / P];
    if (phys < 0 || phys >= num_pages) {
        if (threadIdx.x == 0) set_error(err, GQA_ERR_BAD_PAGE);
        return;
    }
    const bool opens = (t % P) == 0;
    for (int e = threadIdx.x; e < Hk * D; e += blockDim.x) {
        const int kvh = e / D, d = e % D;
        const uint16_t kb = k_new[((size_t)b * Hk + kvh) * D + d];
        uint16_t *dst = kt + (((size_t)phys * Hk + kvh) * D + d) * 2;
        if (opens) {
            dst[0] = kb;
            dst[1] = kb;
        } else {
            const float v = bf16_bits_f32(kb);
            if (v < bf16_bits_f32(dst[0])) dst[0] = kb;
            if (v > bf16_bits_f32(dst[1])) dst[1] = kb;
        }
    }
}

// ---------------------------------------------------------------------------- selection
// Block-wide exclusive prefix sum of one int per thread (kSelThreads threads).
__device__ __forceinline__ int block_exclusive_sum(int v, int *red, int &total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) red[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int w = lane < kSelThreads / 32 ? red[lane] : 0;
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o) wi += t;
        }
        if (lane < kSelThreads / 32) red[lane] = wi - w;  // exclusive warp offsets
        if (lane == 31) red[32] = wi;
    }
    __syncthreads();
    const int r = red[warp] + incl - v;
    total = red[32];
    __syncthreads();
    return r;
}

// First window page of a sequence of L tokens (np pages when the window is empty).
__device__ __forceinline__ int window_first_page(int L, int np, int P, int window) {
    const int lo = L - window > 0 ? L - window : 0;
    return window > 0 ? min(lo / P, np) : np;
}

// Scores of the earlier (non-window) pages, kSelChunk pages per CTA: grid (page chunk,
// kv head, sequence).  The chunk's page-table entries go to shared memory first, then its
// KT rows (every load of a thread issued before the first store), padded to D + 1 words
// per row so that the 32 lanes of a warp, each reading word d of its own page, hit 32
// banks.  One thread per (page, query head) sums that head's D terms in order; one thread
// per page then sums the heads in order.  The scores are written as order-preserving
// keys to keys[(b * Hk + kvh) * pt_stride + page].
template <int D>
__global__ void __launch_bounds__(kSelThreads) sparse_score_kernel(
    const uint16_t *__restrict__ q, const uint32_t *__restrict__ kt,
    const int32_t *__restrict__ page_table, int pt_stride, const int32_t *__restrict__ seq_lens,
    int Hq, int Hk, int P, int num_pages, int topk, int window, uint32_t *__restrict__ keys,
    int *err) {
    constexpr int RW = D + 1;
    constexpr int kWords = kSelChunk * D / kSelThreads;  // KT words each thread stages
    __shared__ float qs[kSparseMaxGroup * D];
    __shared__ uint32_t stage[kSelChunk * RW];
    __shared__ float part[kSparseMaxGroup * kSelChunk];
    __shared__ int phys_s[kSelChunk];
    const int g = Hq / Hk;
    const int kvh = blockIdx.y, b = blockIdx.z;
    const int c0 = blockIdx.x * kSelChunk;
    // launched with programmatic stream serialization: no input or output is touched before
    // the previous kernel in the stream is complete; the pick kernel may become resident
    grid_dependency_wait();
    grid_dependents_launch();
    int L = seq_lens[b];
    if (L < 0 || L > pt_stride * P) L = L < 0 ? 0 : pt_stride * P;  // reported by the pick kernel
    const int np = (L + P - 1) / P;
    const int wp = window_first_page(L, np, P, window);
    if (wp <= topk || c0 >= wp) return;  // uniform for the CTA: nothing to score here
    const int cn = min(kSelChunk, wp - c0);
    for (int e = threadIdx.x; e < g * D; e += kSelThreads)
        qs[e] = bf16_bits_f32(q[((size_t)b * Hq + kvh * g) * D + e]);
    if (threadIdx.x < cn) {
        int ph = page_table[(size_t)b * pt_stride + c0 + threadIdx.x];
        if (ph < 0 || ph >= num_pages) {
            set_error(err, GQA_ERR_BAD_PAGE);
            ph = -1;  // scores as an all-zero box
        }
        phys_s[threadIdx.x] = ph;
    }
    __syncthreads();
    uint32_t w[kWords];
#pragma unroll
    for (int k = 0; k < kWords; ++k) {
        const int e = threadIdx.x + k * kSelThreads;
        const int i = e / D, d = e % D;
        const int ph = i < cn ? phys_s[i] : -1;
        w[k] = ph >= 0 ? __ldg(kt + ((size_t)ph * Hk + kvh) * D + d) : 0u;
    }
#pragma unroll
    for (int k = 0; k < kWords; ++k) {
        const int e = threadIdx.x + k * kSelThreads;
        stage[(e / D) * RW + e % D] = w[k];
    }
    __syncthreads();
    for (int e = threadIdx.x; e < g * kSelChunk; e += kSelThreads) {
        const int i = e % kSelChunk, h = e / kSelChunk;
        if (i >= cn) continue;
        const float *qh = qs + h * D;
        const uint32_t *r = stage + i * RW;
        float sh = 0.f;
#pragma unroll 8
        for (int d = 0; d < D; ++d) {
            const uint32_t x = r[d];
            const float lo = qh[d] * bf16_bits_f32(x & 0xffffu);
            const float hi = qh[d] * bf16_bits_f32(x >> 16);
            sh = __fadd_rn(sh, lo > hi ? lo : hi);
        }
        part[h * kSelChunk + i] = sh;
    }
    __syncthreads();
    if (threadIdx.x < cn) {
        float tot = 0.f;
        for (int h = 0; h < g; ++h) tot = __fadd_rn(tot, part[h * kSelChunk + threadIdx.x]);
        keys[((size_t)b * Hk + kvh) * pt_stride + c0 + threadIdx.x] = score_key(tot);
    }
}

// The choice per (kv head, sequence), one CTA each: the `topk` largest keys among the
// earlier pages by radix select (8 bits a pass, most significant first; each pass a
// histogram in shared memory and a warp scan over its 256 bins), the lowest pages first
// among keys equal to the threshold, plus the window pages; then the chosen pages in
// ascending order as physical * Hk + kvh, and their token count.
__global__ void __launch_bounds__(kSelThreads) sparse_pick_kernel(
    const uint32_t *__restrict__ keys_g, const int32_t *__restrict__ page_table, int pt_stride,
    const int32_t *__restrict__ seq_lens, int Hk, int P, int num_pages, int topk, int window,
    int32_t *__restrict__ sel_table, int sel_stride, int32_t *__restrict__ sel_lens,
    int32_t *__restrict__ sel_pages, int *err) {
    extern __shared__ __align__(16) uint8_t smem[];
    uint32_t *keys = reinterpret_cast<uint32_t *>(smem);           // [pt_stride]
    int *hist = reinterpret_cast<int *>(keys + pt_stride);         // [256]
    int *red = hist + 256;                                         // [40]
    uint8_t *take = reinterpret_cast<uint8_t *>(red + 40);         // [pt_stride]
    __shared__ uint32_t s_prefix;
    __shared__ int s_remaining;
    const int kvh = blockIdx.x, b = blockIdx.y;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const size_t row = (size_t)b * Hk + kvh;
    // behind the score kernel, with programmatic stream serialization: the keys are read
    // once it is complete; the decode of the chosen pages may become resident
    grid_dependency_wait();
    grid_dependents_launch();
    int L = seq_lens[b];
    if (L < 0 || L > pt_stride * P) {
        if (threadIdx.x == 0 && kvh == 0) set_error(err, GQA_ERR_BAD_PAGE);
        L = L < 0 ? 0 : pt_stride * P;
    }
    const int np = (L + P - 1) / P;
    const int wp = window_first_page(L, np, P, window);
    const int32_t *pt = page_table + (size_t)b * pt_stride;
    const bool dense = wp <= topk;
    for (int p = threadIdx.x; p < np; p += blockDim.x) take[p] = (dense || p >= wp) ? 1 : 0;
    if (!dense) {
        for (int p = threadIdx.x; p < wp; p += blockDim.x) keys[p] = keys_g[row * pt_stride + p];
        if (threadIdx.x == 0) {
            s_prefix = 0u;
            s_remaining = topk;
        }
        uint32_t mask = 0u;
        for (int shift = 24; shift >= 0; shift -= 8) {
            for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
            __syncthreads();
            const uint32_t prefix = s_prefix;
            for (int p = threadIdx.x; p < wp; p += blockDim.x) {
                const uint32_t k = keys[p];
                if ((k & mask) == prefix) atomicAdd(&hist[(k >> shift) & 0xffu], 1);
            }
            __syncthreads();
            if (warp == 0) {
                // lane l holds bins 255 - 8l ... 248 - 8l (descending); find the bin where the
                // count from the top first reaches the remaining number
                const int rem = s_remaining;
                int cnt[8], sum = 0;
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    cnt[k] = hist[255 - 8 * lane - k];
                    sum += cnt[k];
                }
                int incl = sum;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int t = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += t;
                }
                const unsigned hit = __ballot_sync(0xffffffffu, incl >= rem);
                const int lw = hit ? __ffs(hit) - 1 : 31;
                if (lane == lw) {
                    int r = rem - (incl - sum), d = 255 - 8 * lane;
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        if (cnt[k] >= r || k == 7) {
                            d = 255 - 8 * lane - k;
                            break;
                        }
                        r -= cnt[k];
                    }
                    s_prefix = prefix | ((uint32_t)d << shift);
                    s_remaining = r;
                }
            }
            mask |= 0xffu << shift;
            __syncthreads();
        }
        const uint32_t T = s_prefix;
        const int need_eq = s_remaining;
        // pages above T are taken; of those equal to T, the first need_eq in page order
        const int per = (wp + kSelThreads - 1) / kSelThreads;
        const int p0 = min(wp, (int)threadIdx.x * per), p1 = min(wp, p0 + per);
        int eq = 0;
        for (int p = p0; p < p1; ++p) eq += keys[p] == T;
        int eq_total;
        int eq_before = block_exclusive_sum(eq, red, eq_total);
        for (int p = p0; p < p1; ++p) {
            const uint32_t k = keys[p];
            if (k > T) take[p] = 1;
            else if (k == T) take[p] = (eq_before++ < need_eq) ? 1 : 0;
        }
    }
    __syncthreads();

    // ---- compaction in ascending page order
    const int per = (np + kSelThreads - 1) / kSelThreads;
    const int p0 = min(np, (int)threadIdx.x * per), p1 = min(np, p0 + per);
    int cnt = 0;
    for (int p = p0; p < p1; ++p) cnt += take[p];
    int total;
    int pos = block_exclusive_sum(cnt, red, total);
    for (int p = p0; p < p1; ++p) {
        if (!take[p]) continue;
        if (pos < sel_stride) {
            const int phys = pt[p];
            const bool ok = phys >= 0 && phys < num_pages;
            if (!ok) set_error(err, GQA_ERR_BAD_PAGE);
            sel_table[row * sel_stride + pos] = ok ? phys * Hk + kvh : 0;
            if (sel_pages) sel_pages[row * sel_stride + pos] = p;
        } else {
            set_error(err, GQA_ERR_SHAPE);
        }
        ++pos;
    }
    if (threadIdx.x == 0) {
        const int n = min(total, sel_stride);
        int tokens = 0;
        if (n > 0) tokens = (np > 0 && take[np - 1] && total <= sel_stride)
                                ? (n - 1) * P + (L - (np - 1) * P)
                                : n * P;
        sel_lens[row] = tokens;
    }
}

}  // namespace

cudaError_t launch_kt_build(const void *k_pages, const int32_t *page_table, int pt_stride,
                            const int32_t *seq_lens, int B, int Hk, int D, int P, int num_pages,
                            void *kt, int *err, cudaStream_t stream) {
    if (B == 0) return cudaSuccess;
    kt_build_kernel<<<dim3(pt_stride, B), 256, 0, stream>>>(
        static_cast<const uint16_t *>(k_pages), page_table, pt_stride, seq_lens, Hk, D, P,
        num_pages, static_cast<uint16_t *>(kt), err);
    return cudaGetLastError();
}

cudaError_t launch_kt_append(const void *k_new, const int32_t *page_table, int pt_stride,
                             const int32_t *seq_lens, int B, int Hk, int D, int P, int num_pages,
                             void *kt, int *err, cudaStream_t stream) {
    if (B == 0) return cudaSuccess;
    kt_append_kernel<<<B, 256, 0, stream>>>(static_cast<const uint16_t *>(k_new), page_table,
                                            pt_stride, seq_lens, Hk, D, P, num_pages,
                                            static_cast<uint16_t *>(kt), err);
    return cudaGetLastError();
}

size_t sparse_pick_smem_bytes(int pt_stride) {
    return sizeof(uint32_t) * (size_t)pt_stride + sizeof(int) * (256 + 40) + (size_t)pt_stride + 16;
}

cudaError_t launch_sparse_select(const void *q, const void *kt, const int32_t *page_table,
                                 int pt_stride, const int32_t *seq_lens, int B, int Hq, int Hk,
                                 int D, int P, int num_pages, int topk, int window,
                                 int32_t *sel_table, int sel_stride, int32_t *sel_lens,
                                 int32_t *sel_pages, uint32_t *keys, int *err,
                                 cudaStream_t stream) {
    if (B == 0) return cudaSuccess;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t sc = {};
    sc.gridDim = dim3((pt_stride + kSelChunk - 1) / kSelChunk, Hk, B);
    sc.blockDim = dim3(kSelThreads);
    sc.stream = stream;
    sc.attrs = attr;
    sc.numAttrs = 1;
    const uint16_t *q16 = static_cast<const uint16_t *>(q);
    const uint32_t *kt32 = static_cast<const uint32_t *>(kt);
    cudaError_t e = D == 128 ? cudaLaunchKernelEx(&sc, sparse_score_kernel<128>, q16, kt32, page_table, pt_stride,
                                                  seq_lens, Hq, Hk, P, num_pages, topk, window, keys, err)
                             : cudaLaunchKernelEx(&sc, sparse_score_kernel<64>, q16, kt32, page_table, pt_stride,
                                                  seq_lens, Hq, Hk, P, num_pages, topk, window, keys, err);
    if (e != cudaSuccess) return e;
    const size_t smem = sparse_pick_smem_bytes(pt_stride);
    e = cudaFuncSetAttribute(sparse_pick_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t pc = sc;
    pc.gridDim = dim3(Hk, B);
    pc.dynamicSmemBytes = smem;
    e = cudaLaunchKernelEx(&pc, sparse_pick_kernel, static_cast<const uint32_t *>(keys), page_table, pt_stride,
                           seq_lens, Hk, P, num_pages, topk, window, sel_table, sel_stride, sel_lens,
                           sel_pages, err);
    return e;
}

}  // namespace gqa
