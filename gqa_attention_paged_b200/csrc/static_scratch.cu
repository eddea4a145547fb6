// static_scratch.cu -- paged GQA decode for callers that cannot allocate device memory.
//
// gqa_paged_decode() takes its scratch (error word, split partials) from a workspace the
// caller allocates.  gqa_paged_decode_static_scratch() runs the same decode with that
// scratch in a fixed array compiled into this library instead, so the caller passes only
// its inputs and outputs.  The array's device address is looked up once per device with
// cudaGetSymbolAddress (the array's name is only a host-side stand-in in host code), and
// the call then goes through gqa_paged_decode() unchanged.
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "gqa_internal.h"
#include "gqa_paged.h"

namespace {

// Scratch shared by every call of gqa_paged_decode_static_scratch on a device.  Every
// GPU that loads this library holds these bytes until the process exits.
static __device__ __align__(256) unsigned char g_static_scratch[GQA_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 128;
std::mutex g_lock;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of g_static_scratch on the current device (looked up on first use).
int scratch_address(void **addr) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return GQA_ERR_LAUNCH;
    std::lock_guard<std::mutex> guard(g_lock);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr)
            return GQA_ERR_LAUNCH;
        g_scratch_addr[dev] = p;
    }
    *addr = g_scratch_addr[dev];
    return GQA_OK;
}

}  // namespace

extern "C" int gqa_paged_decode_static_scratch(
    const void *q, const void *k_pages, const void *v_pages, const float *k_scale,
    const float *v_scale, int kv_dtype, const int32_t *page_table, int pt_stride,
    const int32_t *seq_lens, int B, int Hq, int Hk, int head_dim, int page_size, int num_pages,
    float scale, int num_splits, int pack_gqa, void *out, float *lse, cudaStream_t stream) {
    // gqa_paged_decode()'s own argument checks first, so a call it would reject queues
    // nothing (not even the memset below); then the size check: the scratch this call
    // needs must fit the fixed array.
    const int chk = gqa::decode_check_args(q, k_pages, v_pages, k_scale, v_scale, kv_dtype,
                                           page_table, pt_stride, seq_lens, B, Hq, Hk, head_dim,
                                           page_size, num_pages, num_splits, out, lse);
    if (chk != GQA_OK) return chk;
    const size_t need = gqa_paged_decode_workspace_size(B, Hq, Hk, head_dim, page_size,
                                                        pt_stride * page_size, kv_dtype,
                                                        num_splits);
    if (need > (size_t)GQA_STATIC_SCRATCH_BYTES) return GQA_ERR_WORKSPACE;
    if (B == 0) return GQA_OK;
    void *ws = nullptr;
    const int st = scratch_address(&ws);
    if (st != GQA_OK) return st;
    // The array keeps the previous call's contents.  What must start at zero is cleared:
    // the error word and the balanced schedule's merge counters (split partials and merge
    // pieces are fully rewritten by every call that reads them).
    size_t zero = gqa::decode_zero_prefix_bytes(B, Hq);
    if (zero > (size_t)GQA_STATIC_SCRATCH_BYTES) zero = (size_t)GQA_STATIC_SCRATCH_BYTES;
    if (cudaMemsetAsync(ws, 0, zero, stream) != cudaSuccess) return GQA_ERR_LAUNCH;
    return gqa_paged_decode(q, k_pages, v_pages, k_scale, v_scale, kv_dtype, page_table,
                            pt_stride, seq_lens, B, Hq, Hk, head_dim, page_size, num_pages, scale,
                            num_splits, pack_gqa, out, lse, ws, (size_t)GQA_STATIC_SCRATCH_BYTES,
                            stream);
}
