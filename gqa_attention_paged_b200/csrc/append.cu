// append.cu -- writes each sequence's new token into the paged KV cache, the step before
// decode ("FasterTransformer source tour": the fused decoder step counts writing the new
// token's K/V into the cache among its three global accesses).
//
// seq_lens[b] already counts the new token, so it goes to position L_b - 1: page
// page_table[b][(L_b - 1) / P], slot (L_b - 1) % P, for every kv head.  bf16 pools take
// the token's bits.  e4m3 pools: a token that opens a page (slot 0) sets that (page, kv
// head)'s scale to absmax / 448 in fp32 (1 for an all-zero token), a later token keeps the
// page's scale, and every element is stored as e4m3(x / scale) (the fp32 quotient rounded
// to nearest even, saturated at +-448), so the page's scale stays per-(page, kv head) as
// decode reads it ("解锁GQA性能潜力…", FP8).
// One CTA per (sequence, kv head), one thread per element.
#include <cuda_fp8.h>

#include "gqa_device.cuh"
#include "gqa_internal.h"

namespace gqa {
namespace {

// Largest |x| of the block's values (blockDim.x = D threads, D a multiple of 32).
__device__ __forceinline__ float block_absmax(float x, float *red) {
    float m = fabsf(x);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = m;
    __syncthreads();
    float r = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) r = fmaxf(r, red[w]);
    return r;
}

__global__ void __launch_bounds__(128) append_kernel(const AppendArgs a) {
    __shared__ float red[2][4];
    const int b = blockIdx.x, kvh = blockIdx.y, d = threadIdx.x;
    // launched with programmatic stream serialization: nothing is read or written before the
    // previous kernel in the stream is complete; the decode behind it may become resident
    grid_dependency_wait();
    grid_dependents_launch();
    const int L = a.seq_lens[b];
    if (L <= 0) return;  // uniform for the CTA
    if (L > a.pt_stride * a.P) {
        if (d == 0 && kvh == 0) set_error(a.err, GQA_ERR_BAD_PAGE);
        return;
    }
    const int t = L - 1;
    const int phys = a.page_table[(size_t)b * a.pt_stride + t / a.P];
    if (phys < 0 || phys >= a.num_pages) {
        if (d == 0 && kvh == 0) set_error(a.err, GQA_ERR_BAD_PAGE);
        return;
    }
    const int slot = t % a.P;
    const size_t src = ((size_t)b * a.Hk + kvh) * a.D + d;
    const size_t dst = (((size_t)phys * a.Hk + kvh) * a.P + slot) * a.D + d;
    const uint16_t kb = reinterpret_cast<const uint16_t *>(a.k_new)[src];
    const uint16_t vb = reinterpret_cast<const uint16_t *>(a.v_new)[src];
    if (a.kv_dtype == GQA_KV_BF16) {
        reinterpret_cast<uint16_t *>(a.k_pages)[dst] = kb;
        reinterpret_cast<uint16_t *>(a.v_pages)[dst] = vb;
        return;
    }
    const float kx = __uint_as_float((uint32_t)kb << 16), vx = __uint_as_float((uint32_t)vb << 16);
    const size_t si = (size_t)phys * a.Hk + kvh;
    float ks, vs;
    if (slot == 0) {
        const float km = block_absmax(kx, red[0]), vm = block_absmax(vx, red[1]);
        ks = km > 0.f ? km / 448.f : 1.f;
        vs = vm > 0.f ? vm / 448.f : 1.f;
        if (d == 0) {
            a.k_scale[si] = ks;
            a.v_scale[si] = vs;
        }
    } else {
        ks = a.k_scale[si];
        vs = a.v_scale[si];
    }
    reinterpret_cast<uint8_t *>(a.k_pages)[dst] =
        (uint8_t)__nv_cvt_float_to_fp8(kx / ks, __NV_SATFINITE, __NV_E4M3);
    reinterpret_cast<uint8_t *>(a.v_pages)[dst] =
        (uint8_t)__nv_cvt_float_to_fp8(vx / vs, __NV_SATFINITE, __NV_E4M3);
}

}  // namespace

cudaError_t launch_append(const AppendArgs &a, cudaStream_t stream) {
    if (a.B == 0) return cudaSuccess;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.B, a.Hk);
    cfg.blockDim = dim3(a.D);
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, append_kernel, a);
}

}  // namespace gqa
