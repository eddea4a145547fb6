// gather.cu -- bit-exact copy-out of the paged cache into contiguous per-sequence
// storage: token t of sequence b lives in logical page t / P at slot t % P, found
// through the page table ("TensorRT-LLM与TensorRT核心差异解析", section 4.2.2
// PageAttention: logically contiguous, physically scattered, mapped by a page table).
// One thread per 16-byte chunk of a (token, kv head) row.
#include "gqa_device.cuh"
#include "gqa_internal.h"

namespace gqa {
namespace {

__global__ void __launch_bounds__(256) gather_kernel(const uint8_t *__restrict__ kp,
                                                     const uint8_t *__restrict__ vp,
                                                     const int32_t *__restrict__ page_table,
                                                     int pt_stride, const int32_t *__restrict__ seq_lens,
                                                     const int64_t *__restrict__ cu_kv, int Hk, int P,
                                                     int num_pages, int row_bytes,
                                                     uint8_t *__restrict__ ko, uint8_t *__restrict__ vo) {
    const int b = blockIdx.y;
    int L = seq_lens[b];
    L = L < 0 ? 0 : (L > pt_stride * P ? pt_stride * P : L);
    const int chunks = row_bytes / 16;
    const int64_t total = (int64_t)L * Hk * chunks;
    const int64_t out0 = cu_kv[b];
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int ch = (int)(i % chunks);
        const int64_t r = i / chunks;
        const int kvh = (int)(r % Hk);
        const int t = (int)(r / Hk);
        const int phys = __ldg(page_table + (size_t)b * pt_stride + t / P);
        if (phys < 0 || phys >= num_pages) continue;
        const size_t src = (((size_t)phys * Hk + kvh) * P + t % P) * row_bytes + (size_t)ch * 16;
        const size_t dst = (((size_t)out0 + t) * Hk + kvh) * row_bytes + (size_t)ch * 16;
        *reinterpret_cast<uint4 *>(ko + dst) = __ldg(reinterpret_cast<const uint4 *>(kp + src));
        *reinterpret_cast<uint4 *>(vo + dst) = __ldg(reinterpret_cast<const uint4 *>(vp + src));
    }
}

}  // namespace

cudaError_t launch_gather(const void *k_pages, const void *v_pages, const int32_t *page_table,
                          int pt_stride, const int32_t *seq_lens, const int64_t *cu_kv, int B,
                          int Hk, int D, int P, int num_pages, int elem_bytes, void *k_out,
                          void *v_out, cudaStream_t stream) {
    const int row_bytes = D * elem_bytes;
    const int64_t per_seq = (int64_t)pt_stride * P * Hk * (row_bytes / 16);
    const int threads = 256;
    int64_t bx = (per_seq + threads - 1) / threads;
    if (bx > 4096) bx = 4096;
    if (bx < 1) bx = 1;
    dim3 grid((unsigned)bx, B);
    gather_kernel<<<grid, threads, 0, stream>>>(
        static_cast<const uint8_t *>(k_pages), static_cast<const uint8_t *>(v_pages), page_table,
        pt_stride, seq_lens, cu_kv, Hk, P, num_pages, row_bytes, static_cast<uint8_t *>(k_out),
        static_cast<uint8_t *>(v_out));
    return cudaGetLastError();
}

}  // namespace gqa
