// prefill.cu -- causal chunked prefill over a paged KV cache on sm_100a tensor cores.
//
// A chunk of Lq new query tokens per sequence is appended after a paged prior context
// ("TensorRT对Grouped Query Attention的支持进展", section "与动态批处理协同": chunked
// prefill); its K/V are already the last Lq cached tokens, and query row i (position
// L - Lq + i) attends to keys 0 .. L - Lq + i.
//
// One CTA = (query tile, kv head, sequence).  The tile packs the g query heads of the
// group with T = 128 / g tokens into 128 rows, row r = (token r / g, head r % g)
// (PackGQA: "解锁GQA性能潜力：从批量大小敏感性到高效优化实践", PackGQA / NumSplits
// section), so each K/V tile feeds every head of the group.  The attention itself is the
// tiled fused form ("TensorRT-LLM与TensorRT核心差异解析", section 4.2.1): per tile of 128
// keys, S = Q K^T on tcgen05 into tensor memory, an fp32 online softmax in registers,
// P (bf16) into shared memory, and O += P V on tcgen05 into tensor memory.
//
// Warp roles (192 threads):
//   warp 0   TMA producer: Q tile (3-D map over [total_q][Hq][D]), then K/V tiles, 16
//            keys per copy, gathered page by page through the page table (2-stage ring).
//   warp 1   allocates tensor memory (S: 128 columns, O: 128 columns) and issues the MMAs
//            (one thread), S_{j+1} overlapping the softmax of tile j.
//   warps 2-5 softmax / correction / epilogue: thread = one row (tensor-memory lane).
// P is written as a bf16 value plus its bf16 residual and O += P_hi V + P_lo V, so the
// probabilities keep ~16 significant bits (a single bf16 P loses up to 2^-9 of each
// weight, visible as ~5e-3 errors in short rows whose terms cancel).
// The running max is only moved when a row's max grows by more than 2^8, so O (kept in
// tensor memory) is rescaled rarely; the final O / l is exact for any reference max.
// Every wait is bounded; on expiry the kernel records GQA_ERR_TIMEOUT, finishes its
// outstanding copies and MMAs (bounded), frees its tensor memory and returns.
#include "gqa_device.cuh"
#include "gqa_internal.h"

namespace gqa {
namespace {

constexpr int kM = 128;                // packed query rows per tile
constexpr int kN = 128;                // keys per KV tile
constexpr int kD = 128;                // head dim
constexpr int kStages = 2;             // K/V ring depth
constexpr int kThreadsP = 192;
constexpr int kHalfBytes = kM * 128;   // one 64-column (128-byte) half of a 128-row tile
constexpr int kTileBytesP = 2 * kHalfBytes;
constexpr int kChunk = 16;             // keys per TMA copy (one box)
constexpr int kChunkBytes = kChunk * 128;
constexpr float kLog2eP = 1.4426950408889634f;
constexpr float kLn2P = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr unsigned kAll = 0xffffffffu;

struct alignas(1024) PSmem {
    uint8_t q[kTileBytesP];
    uint8_t k[kStages][kTileBytesP];
    uint8_t v[kStages][kTileBytesP];
    uint8_t p[kTileBytesP];     // bf16 part of P
    uint8_t p_lo[kTileBytesP];  // bf16 residual of P (P - p): two MMAs keep P at ~16 bits
    uint64_t q_full;
    uint64_t kv_full[kStages];
    uint64_t kv_empty[kStages];
    uint64_t s_full, s_free, p_full, pv_done, mma_done;
    uint32_t tmem_base;
    int abort_flag;
};

__device__ __forceinline__ bool wait_all(uint64_t *bar, uint32_t parity) {
    const bool ok = mbar_wait(bar, parity);
    return !__any_sync(kAll, !ok);
}

__global__ void __launch_bounds__(kThreadsP, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                   const __grid_constant__ CUtensorMap qmap, const PrefillArgs a, const int T) {
    extern __shared__ uint8_t smem_raw[];
    PSmem &sm = *reinterpret_cast<PSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.z, kvh = blockIdx.y;
    const int qt = gridDim.x - 1 - blockIdx.x;  // longest (latest) tiles first
    const int g = a.Hq / a.Hk;
    const int q0 = a.cu_q[b];
    const int Lq = a.cu_q[b + 1] - q0;
    const int i0 = qt * T;
    if (blockIdx.x == 0 && threadIdx.x == 0 && Lq > (int)gridDim.x * T)
        set_error(a.err, GQA_ERR_SHAPE);  // max_q_len below a chunk length
    if (i0 >= Lq) return;  // uniform for the whole CTA
    int L = a.seq_lens[b];
    const int P = a.P;
    if (L < Lq || L > a.pt_stride * P) {
        if (threadIdx.x == 0) set_error(a.err, GQA_ERR_BAD_PAGE);
        return;
    }
    const int ntok = min(T, Lq - i0);
    const int rows_valid = ntok * g;
    const int pos_hi = L - Lq + i0 + ntok - 1;
    const int n_kv = a.causal ? pos_hi / kN + 1 : (L + kN - 1) / kN;

    if (threadIdx.x == 0) {
        mbar_init(&sm.q_full, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.kv_full[s], 1);
            mbar_init(&sm.kv_empty[s], 1);
        }
        mbar_init(&sm.s_full, 1);
        mbar_init(&sm.s_free, 4);
        mbar_init(&sm.p_full, 4);
        mbar_init(&sm.pv_done, 1);
        mbar_init(&sm.mma_done, 1);
        sm.abort_flag = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, 256);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = sm.tmem_base;
    const uint32_t tS = tmem, tO = tmem + 128;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        const uint64_t pol_kv = policy_evict_last();  // K/V are re-read by the other q tiles
        if (lane == 0) {
            prefetch_tensormap(&qmap);
            prefetch_tensormap(&kmap);
            prefetch_tensormap(&vmap);
            mbar_arrive_expect_tx(&sm.q_full, 2 * g * T * 128);
            tma_load_3d(sm.q, &qmap, &sm.q_full, 0, kvh * g, q0 + i0, policy_evict_first());
            tma_load_3d(sm.q + kHalfBytes, &qmap, &sm.q_full, 64, kvh * g, q0 + i0,
                        policy_evict_first());
        }
        const int32_t *pt = a.page_table + (size_t)b * a.pt_stride;
        int issued = 0;
        bool fail = false;
        for (int j = 0; j < n_kv && !fail; ++j) {
            const int stage = j % kStages, use = j / kStages;
            const int key0 = j * kN + kChunk * lane;
            int row = -1;
            if (lane < kN / kChunk && key0 < L) {
                const int phys = __ldg(pt + key0 / P);
                if (phys >= 0 && phys < a.num_pages)
                    row = (phys * a.Hk + kvh) * P + key0 % P;
                else
                    set_error(a.err, GQA_ERR_BAD_PAGE);
            }
            const unsigned mask = __ballot_sync(kAll, row >= 0);
            int rows[kN / kChunk];
#pragma unroll
            for (int c = 0; c < kN / kChunk; ++c) rows[c] = __shfl_sync(kAll, row, c);
            if (lane == 0) {
                if (use > 0 && !mbar_wait(&sm.kv_empty[stage], (use - 1) & 1)) {
                    set_error(a.err, GQA_ERR_TIMEOUT);
                    fail = true;
                } else {
                    mbar_arrive_expect_tx(&sm.kv_full[stage], __popc(mask) * 4 * kChunkBytes);
#pragma unroll
                    for (int c = 0; c < kN / kChunk; ++c) {
                        if (!((mask >> c) & 1u)) continue;
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            tma_load_2d(sm.k[stage] + h * kHalfBytes + c * kChunkBytes, &kmap,
                                        &sm.kv_full[stage], 64 * h, rows[c], pol_kv);
                            tma_load_2d(sm.v[stage] + h * kHalfBytes + c * kChunkBytes, &vmap,
                                        &sm.kv_full[stage], 64 * h, rows[c], pol_kv);
                        }
                    }
                    issued = j + 1;
                }
            }
            fail = __shfl_sync(kAll, fail, 0);
        }
        if (lane == 0) {
            // no copy may outlive the CTA: wait for the Q tile and the last issued tiles
            if (!mbar_wait(&sm.q_full, 0)) set_error(a.err, GQA_ERR_TIMEOUT);
            for (int j = max(0, issued - kStages); j < issued; ++j)
                if (!mbar_wait(&sm.kv_full[j % kStages], (j / kStages) & 1)) {
                    set_error(a.err, GQA_ERR_TIMEOUT);
                    break;
                }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        constexpr uint32_t idesc_qk = idesc_bf16_f32(kM, kN, 0, 0);   // Q, K both K-major
        constexpr uint32_t idesc_pv = idesc_bf16_f32(kM, kD, 0, 1);   // P K-major, V MN-major
        const uint32_t qa = smem_u32(sm.q), pa = smem_u32(sm.p), pla = smem_u32(sm.p_lo);
        bool ok = wait_all(&sm.q_full, 0) && wait_all(&sm.kv_full[0], 0);
        int committed_pv = 0;  // PV MMAs committed to pv_done
        if (ok) {
            tc_fence_after_sync();
            if (lane == 0) {
                const uint32_t ka = smem_u32(sm.k[0]);
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
                    tc_mma_ss(tS, smem_desc_sw128(qa + off, 16, 1024),
                              smem_desc_sw128(ka + off, 16, 1024), idesc_qk, kk > 0);
                }
                tc_commit(&sm.s_full);
            }
            __syncwarp();
        }
        for (int j = 0; j < n_kv && ok; ++j) {
            const int stage = j % kStages;
            if (j + 1 < n_kv) {
                ok = wait_all(&sm.kv_full[(j + 1) % kStages], ((j + 1) / kStages) & 1) &&
                     wait_all(&sm.s_free, j & 1);
                if (!ok) break;
                tc_fence_after_sync();
                if (lane == 0) {
                    const uint32_t ka = smem_u32(sm.k[(j + 1) % kStages]);
#pragma unroll
                    for (int kk = 0; kk < kD / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
                        tc_mma_ss(tS, smem_desc_sw128(qa + off, 16, 1024),
                                  smem_desc_sw128(ka + off, 16, 1024), idesc_qk, kk > 0);
                    }
                    tc_commit(&sm.s_full);
                }
                __syncwarp();
            }
            ok = wait_all(&sm.p_full, j & 1);
            if (!ok) break;
            tc_fence_after_sync();
            if (j == n_kv - 1) {
                // keys at or past L hold anything (even NaN): zero those V rows so their
                // zero weights contribute exactly zero.
                const int valid = L - j * kN;
                if (valid < kN) {
                    for (int e = lane; e < (kN - valid) * 16; e += 32) {
                        const int r = valid + (e >> 4), c16 = e & 15;
                        *reinterpret_cast<uint4 *>(sm.v[stage] + (c16 >> 3) * kHalfBytes + r * 128 +
                                                   (c16 & 7) * 16) = make_uint4(0u, 0u, 0u, 0u);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                }
            }
            if (lane == 0) {
                const uint32_t va = smem_u32(sm.v[stage]);
#pragma unroll
                for (int kk = 0; kk < kN / 16; ++kk) {
                    const uint32_t aoff = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
                    tc_mma_ss(tO, smem_desc_sw128(pa + aoff, 16, 1024),
                              smem_desc_sw128(va + kk * 2048, kHalfBytes, 1024), idesc_pv,
                              (j > 0 || kk > 0) ? 1u : 0u);
                }
#pragma unroll
                for (int kk = 0; kk < kN / 16; ++kk) {
                    const uint32_t aoff = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
                    tc_mma_ss(tO, smem_desc_sw128(pla + aoff, 16, 1024),
                              smem_desc_sw128(va + kk * 2048, kHalfBytes, 1024), idesc_pv, 1u);
                }
                tc_commit(&sm.pv_done);
                tc_commit(&sm.kv_empty[stage]);
            }
            committed_pv = j + 1;
            __syncwarp();
        }
        if (!ok && lane == 0) set_error(a.err, GQA_ERR_TIMEOUT);
        (void)committed_pv;
        // every MMA issued must be finished before tensor memory is released
        if (lane == 0) tc_commit(&sm.mma_done);
        __syncwarp();
        if (!wait_all(&sm.mma_done, 0) && lane == 0) set_error(a.err, GQA_ERR_TIMEOUT);
    } else {
        // ------------------------------------------------------------ softmax warps
        const int quad = warp & 3;
        const int row = quad * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        const bool valid_row = row < rows_valid;
        const int tok = i0 + row / g;
        const int hh = row % g;
        const int lim = a.causal ? min(L - Lq + tok, L - 1) : L - 1;  // last visible key
        const float scale_log2 = a.scale * kLog2eP;
        float m_ref = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < n_kv; ++j) {
            if (!wait_all(&sm.s_full, j & 1)) {
                ok = false;
                break;
            }
            tc_fence_after_sync();
            uint32_t sr[4][32];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(tS + lane_off + 32 * c, sr[c]);
            tmem_wait_ld();
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.s_free);

            const int nvis = lim - j * kN + 1;  // keys of this tile the row may see
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const float x = (32 * c + e < nvis) ? __uint_as_float(sr[c][e]) * scale_log2
                                                        : -INFINITY;
                    sr[c][e] = __float_as_uint(x);
                    mx = fmaxf(mx, x);
                }
            const bool need = mx > m_ref + kRescaleThreshold;
            const float new_ref = need ? mx : m_ref;
            const float mref0 = new_ref == -INFINITY ? 0.f : new_ref;
            const float alpha = fast_exp2(m_ref - mref0);

            if (j > 0) {
                if (!wait_all(&sm.pv_done, (j - 1) & 1)) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                if (__any_sync(kAll, need)) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        uint32_t o[32];
                        tmem_ld32(tO + lane_off + 32 * c, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e)
                            o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                        tmem_st32(tO + lane_off + 32 * c, o);
                    }
                    tmem_wait_st();
                }
            }
            // P row (bf16 value + bf16 residual) into the swizzled K-major tiles: 16 chunks
            // of 8 keys each.
            float sum = 0.f;
            uint8_t *prow = sm.p + row * 128;
            uint8_t *plrow = sm.p_lo + row * 128;
#pragma unroll
            for (int ch = 0; ch < 16; ++ch) {
                float pv[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    pv[e] = fast_exp2(__uint_as_float(sr[ch >> 2][(ch & 3) * 8 + e]) - mref0);
                    sum += pv[e];
                }
                uint4 w, wl;
                split_bf16x2(pv[0], pv[1], w.x, wl.x);
                split_bf16x2(pv[2], pv[3], w.y, wl.y);
                split_bf16x2(pv[4], pv[5], w.z, wl.z);
                split_bf16x2(pv[6], pv[7], w.w, wl.w);
                const int off = (ch >> 3) * kHalfBytes + (((ch & 7) ^ (row & 7)) << 4);
                *reinterpret_cast<uint4 *>(prow + off) = w;
                *reinterpret_cast<uint4 *>(plrow + off) = wl;
            }
            l = l * alpha + sum;
            m_ref = new_ref;
            fence_proxy_async_smem();
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.p_full);
        }
        if (ok && wait_all(&sm.pv_done, (n_kv - 1) & 1)) {
            tc_fence_after_sync();
            const float inv = l > 0.f ? 1.f / l : 0.f;
            __nv_bfloat16 *dst = reinterpret_cast<__nv_bfloat16 *>(a.out) +
                                 ((size_t)(q0 + tok) * a.Hq + kvh * g + hh) * kD;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t o[32];
                tmem_ld32(tO + lane_off + 32 * c, o);
                tmem_wait_ld();
                if (valid_row) {
#pragma unroll
                    for (int e = 0; e < 32; e += 8) {
                        uint4 w;
                        w.x = pack_bf16(__uint_as_float(o[e]) * inv, __uint_as_float(o[e + 1]) * inv);
                        w.y = pack_bf16(__uint_as_float(o[e + 2]) * inv, __uint_as_float(o[e + 3]) * inv);
                        w.z = pack_bf16(__uint_as_float(o[e + 4]) * inv, __uint_as_float(o[e + 5]) * inv);
                        w.w = pack_bf16(__uint_as_float(o[e + 6]) * inv, __uint_as_float(o[e + 7]) * inv);
                        *reinterpret_cast<uint4 *>(dst + 32 * c + e) = w;
                    }
                }
            }
            if (valid_row && a.lse)
                a.lse[(size_t)(q0 + tok) * a.Hq + kvh * g + hh] =
                    l > 0.f ? (m_ref + __log2f(l)) * kLn2P : -INFINITY;
        } else if (lane == 0) {
            set_error(a.err, GQA_ERR_TIMEOUT);
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, 256);
    }
}

}  // namespace

cudaError_t launch_prefill(const PrefillArgs &a, const CUtensorMap &kmap, const CUtensorMap &vmap,
                           const CUtensorMap &qmap, cudaStream_t stream) {
    const int g = a.Hq / a.Hk;
    const int T = kM / g;
    const size_t smem = sizeof(PSmem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const int tiles = (a.max_q_len + T - 1) / T;
    if (tiles == 0 || a.B == 0) return cudaSuccess;
    dim3 grid(tiles, a.Hk, a.B);
    prefill_kernel<<<grid, kThreadsP, smem, stream>>>(kmap, vmap, qmap, a, T);
    return cudaGetLastError();
}

}  // namespace gqa
