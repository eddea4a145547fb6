// combine.cu -- log-sum-exp merge of split-KV partial results (NumSplits:
// "解锁GQA性能潜力：从批量大小敏感性到高效优化实践", section
// "核心参数调优：PackGQA与NumSplits的协同舞蹈").  One warp per output row; each lane
// owns D/32 consecutive dims, read as one vector per split.
#include "gqa_device.cuh"
#include "gqa_internal.h"

namespace gqa {
namespace {

constexpr float kLog2e = 1.4426950408889634f;

template <int D, typename OutT>
__global__ void __launch_bounds__(256) lse_combine_kernel(const float *__restrict__ o_part,
                                                          const float *__restrict__ lse_part,
                                                          int num_splits, int rows,
                                                          OutT *__restrict__ out,
                                                          float *__restrict__ lse) {
    constexpr int V = D / 32;
    const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    // launched with programmatic stream serialization: the partials are read only once the
    // kernel that wrote them (the previous one in the stream) has completed
    grid_dependency_wait();
    if (row >= rows) return;
    float M = -INFINITY;
    for (int s = lane; s < num_splits; s += 32) M = fmaxf(M, __ldg(lse_part + (size_t)s * rows + row));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float acc[V];
#pragma unroll
    for (int v = 0; v < V; ++v) acc[v] = 0.f;
    float W = 0.f;
    if (M != -INFINITY) {
        for (int s = 0; s < num_splits; ++s) {
            const float w = exp2f((__ldg(lse_part + (size_t)s * rows + row) - M) * kLog2e);
            if (w > 0.f) {  // empty splits (lse = -inf) contribute nothing, whatever o holds
                const float *src = o_part + ((size_t)s * rows + row) * D + lane * V;
                float x[V];
                if constexpr (V == 4) {
                    float4 t = __ldg(reinterpret_cast<const float4 *>(src));
                    x[0] = t.x; x[1] = t.y; x[2] = t.z; x[3] = t.w;
                } else {
                    float2 t = __ldg(reinterpret_cast<const float2 *>(src));
                    x[0] = t.x; x[1] = t.y;
                }
                W += w;
#pragma unroll
                for (int v = 0; v < V; ++v) acc[v] += w * x[v];
            }
        }
    }
    const float inv = W > 0.f ? 1.f / W : 0.f;
    if constexpr (sizeof(OutT) == 4) {
        float2 *dst = reinterpret_cast<float2 *>(out + (size_t)row * D + lane * V);
#pragma unroll
        for (int v = 0; v < V; v += 2) dst[v / 2] = make_float2(acc[v] * inv, acc[v + 1] * inv);
    } else {
        __nv_bfloat162 *dst = reinterpret_cast<__nv_bfloat162 *>(out + (size_t)row * D + lane * V);
#pragma unroll
        for (int v = 0; v < V; v += 2) dst[v / 2] = __floats2bfloat162_rn(acc[v] * inv, acc[v + 1] * inv);
    }
    if (lane == 0 && lse) lse[row] = W > 0.f ? M + logf(W) : -INFINITY;
}

}  // namespace

cudaError_t launch_lse_combine(const float *o_part, const float *lse_part, int num_splits,
                               int rows, int D, void *out, float *lse, cudaStream_t stream,
                               int out_f32) {
    if (rows <= 0) return cudaSuccess;
    const int threads = 256;
    const int blocks = (int)(((size_t)rows * 32 + threads - 1) / threads);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(blocks);
    cfg.blockDim = dim3(threads);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (out_f32)
        return D == 128 ? cudaLaunchKernelEx(&cfg, lse_combine_kernel<128, float>, o_part, lse_part,
                                             num_splits, rows, static_cast<float *>(out), lse)
                        : cudaLaunchKernelEx(&cfg, lse_combine_kernel<64, float>, o_part, lse_part,
                                             num_splits, rows, static_cast<float *>(out), lse);
    return D == 128 ? cudaLaunchKernelEx(&cfg, lse_combine_kernel<128, __nv_bfloat16>, o_part, lse_part,
                                         num_splits, rows, static_cast<__nv_bfloat16 *>(out), lse)
                    : cudaLaunchKernelEx(&cfg, lse_combine_kernel<64, __nv_bfloat16>, o_part, lse_part,
                                         num_splits, rows, static_cast<__nv_bfloat16 *>(out), lse);
}

}  // namespace gqa
