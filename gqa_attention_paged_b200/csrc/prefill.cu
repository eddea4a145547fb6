// prefill.cu -- causal chunked prefill (tcgen05 / TMEM kernel: not built yet).
#include "gqa_internal.h"
#include "gqa_paged.h"

extern "C" int gqa_paged_prefill(const void *, const int32_t *, const void *, const void *,
                                 const int32_t *, int, const int32_t *, int, int, int, int, int,
                                 int, float, int, int, int, void *, float *, void *, size_t,
                                 cudaStream_t) {
    return GQA_ERR_SHAPE;
}
