// decode.cu -- paged GQA decode kernel for sm_100a (bf16 and fp8-e4m3 KV).
//
// One CTA = (split, kv head [, head chunk], sequence).  It streams the split's KV tiles
// (16 tokens of one page each) from the pool into a shared-memory ring with TMA tile
// loads (128-byte swizzled, no multicast), and computes attention for ALL query heads
// of the group at once (PackGQA: "解锁GQA性能潜力：从批量大小敏感性到高效优化实践",
// section "核心参数调优：PackGQA与NumSplits的协同舞蹈"), so every KV byte crosses HBM
// once.  Scores and P·V run on warp-level tensor cores (m16n8k16, fp32 accumulate) with
// the tokens of a tile as the M dimension and the packed heads as N; the softmax is the
// online (running max / running sum) form in fp32, exp2 domain, as in the tiled fused
// attention of "TensorRT-LLM与TensorRT核心差异解析", section 4.2.1 FlashAttention.
//
// Warp roles: warp 4 is the producer (page-table resolve, TMA issue, one elected lane);
// warps 0..3 are consumers, taking tiles round-robin, each with its own softmax state,
// merged through shared memory at the end.  Every wait is bounded (2 s): on expiry the
// kernel records GQA_ERR_TIMEOUT in the workspace error word and returns.
//
// Tile layout in shared memory (per K or V tile, 16 token rows): the row is cut into
// 128-byte boxes (2 for bf16 D=128, 1 for bf16 D=64 and fp8 D=128); box j of row r sits
// at j*16*128 + r*128, its 16-byte chunks permuted by chunk ^ (r & 7) (the TMA 128B
// swizzle), so ldmatrix reads of 8 rows at one chunk hit 8 different bank groups.
#include "gqa_device.cuh"
#include "gqa_internal.h"

namespace gqa {
namespace {

constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kTile = kDecodeTileTokens;  // tokens per pipeline stage
constexpr unsigned kFull = 0xffffffffu;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

template <int D, bool FP8>
struct Cfg {
    static constexpr int kElt = FP8 ? 1 : 2;
    static constexpr int kRowBytes = D * kElt;
    static constexpr int kBoxes = kRowBytes / 128;     // TMA boxes per tile row
    static constexpr int kBoxCols = 128 / kElt;        // elements per box row
    static constexpr int kTileBytes = kTile * kRowBytes;
    static constexpr int kStageBytes = 2 * kTileBytes;
    static constexpr int kStagesRaw = 65536 / kStageBytes;
    static constexpr int kStages = kStagesRaw < 4 ? 4 : (kStagesRaw > 16 ? 16 : kStagesRaw);
};

template <int D, bool FP8>
struct alignas(1024) Smem {
    uint8_t tiles[Cfg<D, FP8>::kStages][2][Cfg<D, FP8>::kTileBytes];
    uint64_t full[Cfg<D, FP8>::kStages];
    uint64_t empty[Cfg<D, FP8>::kStages];
    float kscale[Cfg<D, FP8>::kStages];
    float vscale[Cfg<D, FP8>::kStages];
    int abort_flag;
};

// Byte offset of (row r, byte cb of the row; cb a multiple of 16) in a swizzled tile.
__device__ __forceinline__ uint32_t swz(int r, int cb) {
    return (uint32_t)((cb >> 7) * (kTile * 128) + r * 128 + ((((cb >> 4) & 7) ^ (r & 7)) << 4));
}

__device__ __forceinline__ void consumer_bar() {
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
}

template <int D, int NT, bool FP8>
__global__ void __launch_bounds__(kThreads, 3)
    decode_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                  const DecodeArgs a, const int heads_per_cta, const int head_chunks) {
    using C = Cfg<D, FP8>;
    constexpr int S = C::kStages;
    constexpr int KT = D / 16;  // 16-wide k steps (scores) and dim tiles (output)
    extern __shared__ uint8_t smem_raw[];
    Smem<D, FP8> &sm = *reinterpret_cast<Smem<D, FP8> *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int split = blockIdx.x;
    const int kvh = blockIdx.y / head_chunks, chunk = blockIdx.y % head_chunks;
    const int b = blockIdx.z;
    const int g = a.Hq / a.Hk;
    const int head_lo = kvh * g + chunk * heads_per_cta;
    const int nh = min(heads_per_cta, g - chunk * heads_per_cta);
    const int P = a.P;

    // This split's token range [t0, t1), page aligned (contiguous ranges of
    // ceil(np / num_splits) pages).
    int L = a.seq_lens[b];
    const int Lmax = a.pt_stride * P;
    if (L < 0 || L > Lmax) {
        if (threadIdx.x == 0) set_error(a.err, GQA_ERR_BAD_PAGE);
        L = L < 0 ? 0 : Lmax;
    }
    const int np = (L + P - 1) / P;
    const int cpp = (np + a.num_splits - 1) / a.num_splits;
    const int t0 = split * cpp * P;
    const int t1 = min(L, (split + 1) * cpp * P);
    const int n_tiles = t1 > t0 ? (t1 - t0 + kTile - 1) / kTile : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        sm.abort_flag = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    __syncthreads();

    if (warp == kConsumerWarps) {
        // ------------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tensormap(&kmap);
            prefetch_tensormap(&vmap);
        }
        const uint64_t pol = a.pack_gqa ? policy_evict_first() : policy_evict_last();
        const int32_t *pt = a.page_table + (size_t)b * a.pt_stride;
        int issued = 0;
        bool fail = false;
        for (int base = 0; base < n_tiles && !fail; base += 32) {
            // Resolve up to 32 tiles' physical pages (and fp8 scales) in one go.
            const int i = base + lane;
            int phys = -1;
            float ksc = 1.f, vsc = 1.f;
            if (i < n_tiles) {
                phys = __ldg(pt + (t0 + i * kTile) / P);
                if (FP8 && phys >= 0 && phys < a.num_pages) {
                    ksc = __ldg(a.k_scale + (size_t)phys * a.Hk + kvh);
                    vsc = __ldg(a.v_scale + (size_t)phys * a.Hk + kvh);
                }
            }
            const int cnt = min(32, n_tiles - base);
            for (int j = 0; j < cnt; ++j) {
                const int it = base + j;
                const int ph = __shfl_sync(kFull, phys, j);
                const float ks = __shfl_sync(kFull, ksc, j);
                const float vs = __shfl_sync(kFull, vsc, j);
                if (lane == 0) {
                    const int stage = it % S, use = it / S;
                    if (use > 0 && !mbar_wait(&sm.empty[stage], (use - 1) & 1)) {
                        set_error(a.err, GQA_ERR_TIMEOUT);
                        fail = true;
                    } else if (ph < 0 || ph >= a.num_pages) {
                        set_error(a.err, GQA_ERR_BAD_PAGE);
                        mbar_arrive(&sm.full[stage]);  // release the stage with stale data
                        issued = it + 1;
                    } else {
                        if (FP8) {
                            sm.kscale[stage] = ks;
                            sm.vscale[stage] = vs;
                        }
                        const int row = (ph * a.Hk + kvh) * P + (t0 + it * kTile) % P;
                        mbar_arrive_expect_tx(&sm.full[stage], 2 * C::kTileBytes);
#pragma unroll
                        for (int bx = 0; bx < C::kBoxes; ++bx) {
                            tma_load_2d(sm.tiles[stage][0] + bx * kTile * 128, &kmap, &sm.full[stage],
                                        bx * C::kBoxCols, row, pol);
                            tma_load_2d(sm.tiles[stage][1] + bx * kTile * 128, &vmap, &sm.full[stage],
                                        bx * C::kBoxCols, row, pol);
                        }
                        issued = it + 1;
                    }
                }
                fail = __shfl_sync(kFull, fail, 0);
                if (fail) break;
            }
        }
        // Drain: the last S issued tiles may still be landing; wait for them (bounded)
        // so no copy into this CTA's shared memory outlives it.
        if (lane == 0) {
            for (int it = max(0, issued - S); it < issued; ++it)
                if (!mbar_wait(&sm.full[it % S], (it / S) & 1)) {
                    set_error(a.err, GQA_ERR_TIMEOUT);
                    break;
                }
        }
        return;
    }

    // -------------------------------------------------------------------- consumers
    const int gq = lane >> 2, cq = lane & 3;  // fragment row group / column pair

    // q as the B operand (k = head dim, n = packed head), registers for the whole CTA.
    uint32_t qf[NT][KT][2];
    float qmul = 1.f;  // fp8 path: power-of-two prescale bringing q into f16 range
    {
        const __nv_bfloat16 *qb = reinterpret_cast<const __nv_bfloat16 *>(a.q);
        if (!FP8) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int hl = nt * 8 + gq;
                const bool ok = hl < nh;
                const uint32_t *qw = reinterpret_cast<const uint32_t *>(
                    qb + ((size_t)b * a.Hq + head_lo + (ok ? hl : 0)) * D);
#pragma unroll
                for (int ks = 0; ks < KT; ++ks) {
                    qf[nt][ks][0] = ok ? __ldg(qw + (ks * 16 + 2 * cq) / 2) : 0u;
                    qf[nt][ks][1] = ok ? __ldg(qw + (ks * 16 + 8 + 2 * cq) / 2) : 0u;
                }
            }
        } else {
            float qv[NT][KT][4];
            float amax = 0.f;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int hl = nt * 8 + gq;
                const bool ok = hl < nh;
                const uint2 *qw = reinterpret_cast<const uint2 *>(
                    qb + ((size_t)b * a.Hq + head_lo + (ok ? hl : 0)) * D);
#pragma unroll
                for (int ks = 0; ks < KT; ++ks) {
                    uint2 w = ok ? __ldg(qw + (ks * 16 + 4 * cq) / 4) : make_uint2(0u, 0u);
                    __nv_bfloat162 lo = *reinterpret_cast<__nv_bfloat162 *>(&w.x);
                    __nv_bfloat162 hi = *reinterpret_cast<__nv_bfloat162 *>(&w.y);
                    qv[nt][ks][0] = __low2float(lo);
                    qv[nt][ks][1] = __high2float(lo);
                    qv[nt][ks][2] = __low2float(hi);
                    qv[nt][ks][3] = __high2float(hi);
#pragma unroll
                    for (int e = 0; e < 4; ++e) amax = fmaxf(amax, fabsf(qv[nt][ks][e]));
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, o));
            if (amax > 0.f && amax < 3.0e38f) {
                int e;
                frexpf(amax, &e);  // amax < 2^e
                qmul = ldexpf(1.f, min(126, 15 - e));
            }
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int ks = 0; ks < KT; ++ks) {
                    qf[nt][ks][0] = pack_f16(qv[nt][ks][0] * qmul, qv[nt][ks][1] * qmul);
                    qf[nt][ks][1] = pack_f16(qv[nt][ks][2] * qmul, qv[nt][ks][3] * qmul);
                }
        }
    }

    float o[NT][KT][4];
    float m[NT][2], l[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int dt = 0; dt < KT; ++dt)
#pragma unroll
            for (int e = 0; e < 4; ++e) o[nt][dt][e] = 0.f;
        m[nt][0] = m[nt][1] = -INFINITY;
        l[nt][0] = l[nt][1] = 0.f;
    }
    const float scale_log2 = a.scale * kLog2e;

    bool fail = false;
    for (int it = warp; it < n_tiles; it += kConsumerWarps) {
        const int stage = it % S;
        const bool ok = mbar_wait(&sm.full[stage], (it / S) & 1);
        if (__any_sync(kFull, !ok)) {
            fail = true;
            break;
        }
        uint8_t *kt = sm.tiles[stage][0];
        uint8_t *vt = sm.tiles[stage][1];
        const int valid = t1 - (t0 + it * kTile);  // >= 1
        if (valid < kTile) {
            // Rows past the end of the sequence may hold anything (even NaN): zero the V
            // rows so 0-weight tokens contribute exactly 0; K rows are masked below.
            constexpr int kChunksPerRow = C::kRowBytes / 16;
            for (int e = lane; e < (kTile - valid) * kChunksPerRow; e += 32) {
                const int r = valid + e / kChunksPerRow, cb = (e % kChunksPerRow) * 16;
                *reinterpret_cast<uint4 *>(vt + swz(r, cb)) = make_uint4(0u, 0u, 0u, 0u);
            }
            __syncwarp();
        }
        const uint32_t kbase = smem_u32(kt), vbase = smem_u32(vt);

        // ---- scores S^T[token][head] = K q^T
        float s[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
        if (!FP8) {
            const int r = (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
            for (int ks = 0; ks < KT; ++ks) {
                uint32_t af[4];
                ldsm_x4(af, kbase + swz(r, (ks * 16 + (lane >> 4) * 8) * 2));
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) mma_bf16(s[nt], af, qf[nt][ks][0], qf[nt][ks][1]);
            }
        } else {
            // One ldmatrix.x4 over 32 fp8 dims serves two k steps; the k order inside a
            // step is permuted identically for K (here) and q (qf), which leaves each dot
            // product unchanged.
            const int j = lane >> 3;
            const int r = (lane & 7) + (j & 1) * 8;
#pragma unroll
            for (int kp = 0; kp < D / 32; ++kp) {
                uint32_t raw[4];
                ldsm_x4(raw, kbase + swz(r, 32 * kp + (j >> 1) * 16));
                uint32_t a0[4] = {e4m3x2_to_f16x2(raw[0] & 0xffff), e4m3x2_to_f16x2(raw[1] & 0xffff),
                                  e4m3x2_to_f16x2(raw[0] >> 16), e4m3x2_to_f16x2(raw[1] >> 16)};
                uint32_t a1[4] = {e4m3x2_to_f16x2(raw[2] & 0xffff), e4m3x2_to_f16x2(raw[3] & 0xffff),
                                  e4m3x2_to_f16x2(raw[2] >> 16), e4m3x2_to_f16x2(raw[3] >> 16)};
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    mma_f16(s[nt], a0, qf[nt][2 * kp][0], qf[nt][2 * kp][1]);
                    mma_f16(s[nt], a1, qf[nt][2 * kp + 1][0], qf[nt][2 * kp + 1][1]);
                }
            }
        }

        // ---- online softmax (exp2 domain), per packed head column
        const float kmul = FP8 ? scale_log2 * sm.kscale[stage] / qmul : scale_log2;
        const bool v0 = gq < valid, v1 = gq + 8 < valid;
        uint32_t pb[NT][2], pbl[NT][2];
        float alpha[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            float p[4];
#pragma unroll
            for (int jj = 0; jj < 2; ++jj) {
                const float x0 = v0 ? s[nt][jj] * kmul : -INFINITY;
                const float x1 = v1 ? s[nt][jj + 2] * kmul : -INFINITY;
                float mx = fmaxf(x0, x1);
                mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 4));
                mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 8));
                mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));
                const float mnew = fmaxf(m[nt][jj], mx);
                const float mref = mnew == -INFINITY ? 0.f : mnew;
                alpha[nt][jj] = fast_exp2(m[nt][jj] - mref);
                p[jj] = fast_exp2(x0 - mref);
                p[jj + 2] = fast_exp2(x1 - mref);
                l[nt][jj] = l[nt][jj] * alpha[nt][jj] + p[jj] + p[jj + 2];
                m[nt][jj] = mnew;
            }
            if (!FP8) {
                // P as a bf16 value plus its bf16 residual: O += V^T P_hi^T + V^T P_lo^T keeps
                // the weights at ~16 bits (one bf16 P would cost up to 2^-9 per weight).
                uint32_t h0, l0, h1, l1;
                split_bf16x2(p[0], p[1], h0, l0);
                split_bf16x2(p[2], p[3], h1, l1);
                pb[nt][0] = movmatrix_trans(h0);
                pb[nt][1] = movmatrix_trans(h1);
                pbl[nt][0] = movmatrix_trans(l0);
                pbl[nt][1] = movmatrix_trans(l1);
            } else {
                pb[nt][0] = movmatrix_trans(pack_f16(p[0], p[1]));
                pb[nt][1] = movmatrix_trans(pack_f16(p[2], p[3]));
            }
#pragma unroll
            for (int dt = 0; dt < KT; ++dt) {
                o[nt][dt][0] *= alpha[nt][0];
                o[nt][dt][1] *= alpha[nt][1];
                o[nt][dt][2] *= alpha[nt][0];
                o[nt][dt][3] *= alpha[nt][1];
            }
        }

        // ---- O^T[dim][head] += V^T P^T
        if (!FP8) {
            const int j = lane >> 3;
            const int r = (lane & 7) + (j >> 1) * 8;
#pragma unroll
            for (int dt = 0; dt < KT; ++dt) {
                uint32_t af[4];
                ldsm_x4_trans(af, vbase + swz(r, (dt * 16 + (j & 1) * 8) * 2));
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    mma_bf16(o[nt][dt], af, pb[nt][0], pb[nt][1]);
                    mma_bf16(o[nt][dt], af, pbl[nt][0], pbl[nt][1]);
                }
            }
        } else {
            // fp8 V: plain ldmatrix gives each lane 4 consecutive dims of one token;
            // after conversion, movmatrix transposes 8x8 blocks into the A layout (dims
            // permuted within each 16-dim tile, undone when O is written out).
            const float vsc = sm.vscale[stage];
            const int j = lane >> 3;
            const int r = (lane & 7) + (j & 1) * 8;
#pragma unroll
            for (int qd = 0; qd < D / 32; ++qd) {
                uint32_t raw[4];
                ldsm_x4(raw, vbase + swz(r, 32 * qd + (j >> 1) * 16));
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const uint32_t lo_t = raw[2 * h], hi_t = raw[2 * h + 1];  // tokens 0-7 / 8-15
                    uint32_t af[4] = {movmatrix_trans(e4m3x2_to_f16x2(lo_t & 0xffff)),
                                      movmatrix_trans(e4m3x2_to_f16x2(lo_t >> 16)),
                                      movmatrix_trans(e4m3x2_to_f16x2(hi_t & 0xffff)),
                                      movmatrix_trans(e4m3x2_to_f16x2(hi_t >> 16))};
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        float pv[4] = {0.f, 0.f, 0.f, 0.f};
                        mma_f16(pv, af, pb[nt][0], pb[nt][1]);
#pragma unroll
                        for (int e = 0; e < 4; ++e) o[nt][2 * qd + h][e] += vsc * pv[e];
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.empty[stage]);
    }

    // ------------------------------------------------------------------ epilogue
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
            float v = l[nt][jj];
            v += __shfl_xor_sync(kFull, v, 4);
            v += __shfl_xor_sync(kFull, v, 8);
            v += __shfl_xor_sync(kFull, v, 16);
            l[nt][jj] = v;
        }
    if (fail && lane == 0) {
        set_error(a.err, GQA_ERR_TIMEOUT);
        sm.abort_flag = 1;
    }
    consumer_bar();  // all tiles consumed: the stage ring is free for the reduction
    if (sm.abort_flag) return;

    constexpr int HW = 8 * NT;  // packed head columns per CTA
    constexpr int RS = D + 4;   // padded row: the 4 lanes sharing a dim hit 4 banks
    float *red_o = reinterpret_cast<float *>(&sm.tiles[0][0][0]);  // [warp][HW][RS]
    float *red_m = red_o + kConsumerWarps * HW * RS;                // [warp][HW]
    float *red_l = red_m + kConsumerWarps * HW;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int h0 = nt * 8 + 2 * cq;
#pragma unroll
        for (int dt = 0; dt < KT; ++dt) {
            int d0, d1;
            if (!FP8) {
                d0 = dt * 16 + gq;
                d1 = d0 + 8;
            } else {
                d0 = dt * 16 + 4 * (gq >> 1) + (gq & 1);
                d1 = d0 + 2;
            }
            float *w = red_o + (size_t)(warp * HW + h0) * RS;
            w[d0] = o[nt][dt][0];
            w[RS + d0] = o[nt][dt][1];
            w[d1] = o[nt][dt][2];
            w[RS + d1] = o[nt][dt][3];
        }
        if (gq == 0) {
            red_m[warp * HW + h0] = m[nt][0];
            red_m[warp * HW + h0 + 1] = m[nt][1];
            red_l[warp * HW + h0] = l[nt][0];
            red_l[warp * HW + h0 + 1] = l[nt][1];
        }
    }
    consumer_bar();

    const size_t rows_total = (size_t)a.B * a.Hq;
    for (int e = threadIdx.x; e < nh * (D / 2); e += kConsumerWarps * 32) {
        const int h = e / (D / 2), d = (e % (D / 2)) * 2;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, red_m[w * HW + h]);
        float Ls = 0.f, o0 = 0.f, o1 = 0.f;
        if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kConsumerWarps; ++w) {
                const float f = fast_exp2(red_m[w * HW + h] - M);
                Ls += f * red_l[w * HW + h];
                o0 += f * red_o[(size_t)(w * HW + h) * RS + d];
                o1 += f * red_o[(size_t)(w * HW + h) * RS + d + 1];
            }
        }
        const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
        const float lse_v = Ls > 0.f ? (M + __log2f(Ls)) * kLn2 : -INFINITY;
        const size_t row = (size_t)b * a.Hq + head_lo + h;
        if (a.num_splits == 1) {
            reinterpret_cast<__nv_bfloat162 *>(a.out)[(row * D + d) / 2] =
                __floats2bfloat162_rn(o0 * inv, o1 * inv);
            if (d == 0 && a.lse) a.lse[row] = lse_v;
        } else {
            const size_t prow = (size_t)split * rows_total + row;
            reinterpret_cast<float2 *>(a.o_part)[(prow * D + d) / 2] = make_float2(o0 * inv, o1 * inv);
            if (d == 0) a.lse_part[prow] = lse_v;
        }
    }
}

template <int D, int NT, bool FP8>
cudaError_t launch_t(const DecodeArgs &a, const CUtensorMap &kmap, const CUtensorMap &vmap,
                     cudaStream_t stream) {
    const size_t smem = sizeof(Smem<D, FP8>) + 1024;
    static_assert(sizeof(float) * kConsumerWarps * 8 * NT * (D + 6) <=
                      sizeof(uint8_t) * Cfg<D, FP8>::kStages * 2 * Cfg<D, FP8>::kTileBytes,
                  "reduction area must fit in the stage ring");
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<D, NT, FP8>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int g = a.Hq / a.Hk;
    const int hpc = a.pack_gqa ? (g < 8 * NT ? g : 8 * NT) : 1;
    const int chunks = (g + hpc - 1) / hpc;
    dim3 grid(a.num_splits, a.Hk * chunks, a.B);
    decode_kernel<D, NT, FP8><<<grid, kThreads, smem, stream>>>(kmap, vmap, a, hpc, chunks);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs &a, const CUtensorMap &kmap, const CUtensorMap &vmap,
                          cudaStream_t stream) {
    const int g = a.Hq / a.Hk;
    const bool wide = a.pack_gqa && g > 8;
    if (a.kv_dtype == GQA_KV_FP8_E4M3) {
        return wide ? launch_t<128, 2, true>(a, kmap, vmap, stream)
                    : launch_t<128, 1, true>(a, kmap, vmap, stream);
    }
    if (a.D == 128)
        return wide ? launch_t<128, 2, false>(a, kmap, vmap, stream)
                    : launch_t<128, 1, false>(a, kmap, vmap, stream);
    return wide ? launch_t<64, 2, false>(a, kmap, vmap, stream)
                : launch_t<64, 1, false>(a, kmap, vmap, stream);
}

}  // namespace gqa
