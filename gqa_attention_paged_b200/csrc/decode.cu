// decode.cu -- paged GQA decode kernels for sm_100a (bf16 and fp8-e4m3 KV).
//
// Both kernels stream 16-token K/V tiles of one page and one kv head from the pool into a
// shared-memory ring with TMA tile loads (128-byte swizzled, no multicast), and compute
// attention for ALL query heads of the group per tile (PackGQA:
// "解锁GQA性能潜力：从批量大小敏感性到高效优化实践", section
// "核心参数调优：PackGQA与NumSplits的协同舞蹈"), so every KV byte crosses HBM once.
// Scores and P·V run on warp-level tensor cores (m16n8k16, fp32 accumulate) with the
// tile's tokens as M and the packed heads as N; the softmax is the online (running max /
// running sum) form in fp32, exp2 domain, as in the tiled fused attention of
// "TensorRT-LLM与TensorRT核心差异解析", section 4.2.1 FlashAttention.
//
// Warp roles: warps 0..3 are consumers; the producer (page-table resolve, TMA issue by one
// lane) is warp 4, except in the e4m3 instances of the balanced kernel, where warps 4..7
// each feed one consumer.  Two schedules share the per-tile code (WarpAttn):
//   - split (decode_kernel): one CTA per (split, kv head [, head chunk], sequence); the
//     split's tiles go round-robin to the 4 warps, merged through shared memory at the
//     end; splits (NumSplits) are merged by lse_combine.
//   - balanced persistent (decode_sk_kernel): a fixed grid; all (sequence, kv head)
//     tiles are laid end to end and every consumer warp takes an equal contiguous share.
//     A warp that holds a whole (sequence, kv head) unit writes its output directly; a
//     unit cut between warps leaves one piece per warp.  The last warp to finish its
//     piece merges them by log-sum-exp in the same launch, or, when units span many
//     warps (a few long sequences), piece_merge_kernel merges every cut unit after it.
// Every wait is bounded (2 s): on expiry the kernel records GQA_ERR_TIMEOUT in the
// workspace error word and returns.
//
// Tile layout in shared memory (per K or V tile, 16 token rows): the row is cut into
// 128-byte boxes (2 for bf16 D=128, 1 for bf16 D=64 and fp8 D=128); box j of row r sits
// at j*16*128 + r*128, its 16-byte chunks permuted by chunk ^ (r & 7) (the TMA 128B
// swizzle), so ldmatrix reads of 8 rows at one chunk hit 8 different bank groups.
#include "gqa_device.cuh"
#include "gqa_internal.h"

namespace gqa {
namespace {

constexpr int kConsumerWarps = kStreamWorkersPerCta;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
// The e4m3 instances of the balanced kernel give every worker its own producer warp (one
// lane of it issues the copies) and move registers to the consumer warpgroup: 4 consumer
// warps at up to 208 registers, 4 producer warps at 40.  The e4m3 tile loop needs the
// registers more than the bf16 one, and its workers no longer wait on one another's
// producer lane (e4m3 B=64 65.3% -> 69.7% of the copy peak, B=128 72.5% -> 77.7%; the bf16
// instances measured faster with one shared producer warp).
constexpr int kThreadsSplitProd = 2 * kConsumerWarps * 32;
constexpr int kRegsProducer = 40, kRegsConsumer = 208;
static_assert(128 * kRegsProducer + 128 * kRegsConsumer <= kThreadsSplitProd * 128,
              "register split of the e4m3 balanced kernel");
template <bool FP8>
constexpr int balanced_threads() { return FP8 ? kThreadsSplitProd : kThreads; }
constexpr unsigned kFull = 0xffffffffu;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLazyRef = 8.0f;  // log2 units a score may pass the reference by

// Ring sizes: the split kernel runs 3 CTAs per SM with a 64 KB ring; the balanced
// kernel runs 2 per SM (more registers per thread) with a 96 KB ring.
constexpr int kRingSplit = 65536;
constexpr int kRingBalanced = 98304;

// TT = tokens per pipeline stage (one TMA box of TT rows of one page and kv head): 16,
// or 32 for e4m3 KV on pages of 32+ tokens (the fp8 tile then carries as many bytes as
// a bf16 one, and two independent 16-token halves per softmax step).
template <int D, bool FP8, int RING = kRingSplit, int TT = 16>
struct Cfg {
    static constexpr int kElt = FP8 ? 1 : 2;
    static constexpr int kRowBytes = D * kElt;
    static constexpr int kBoxes = kRowBytes / 128;     // TMA boxes per tile row
    static constexpr int kBoxCols = 128 / kElt;        // elements per box row
    static constexpr int kTileBytes = TT * kRowBytes;
    static constexpr int kStageBytes = 2 * kTileBytes;
    static constexpr int kStagesRaw = RING / kStageBytes;
    static constexpr int kStages = kStagesRaw < 4 ? 4 : (kStagesRaw > 32 ? 32 : kStagesRaw);
    static_assert(kStages % kConsumerWarps == 0, "stage i belongs to consumer warp i % 4");
};

// Per-stage tile description written by the producer (balanced schedule).
struct TileRec {
    int b;       // sequence, or -1 for an empty slot
    int y;       // unit within the sequence: kv head * head chunks + chunk
    int tile;    // tile index within the unit
    int valid;   // tokens of the tile inside the sequence
    long long f; // flat tile index
};

template <int D, bool FP8, int RING = kRingSplit, int TT = 16>
struct alignas(1024) Smem {
    using C = Cfg<D, FP8, RING, TT>;
    uint8_t tiles[C::kStages][2][C::kTileBytes];
    uint64_t full[C::kStages];
    uint64_t empty[C::kStages];
    float kscale[C::kStages][2];  // per 16-token half of the tile
    float vscale[C::kStages][2];
    TileRec rec[C::kStages];
    int abort_flag;
};

// Byte offset of (row r, byte cb of the row; cb a multiple of 16) in a swizzled tile of
// TT rows.
template <int TT>
__device__ __forceinline__ uint32_t swz(int r, int cb) {
    return (uint32_t)((cb >> 7) * (TT * 128) + r * 128 + ((((cb >> 4) & 7) ^ (r & 7)) << 4));
}

__device__ __forceinline__ void consumer_bar() {
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
}

// Adds `bytes` to the barrier's expected transaction count without an arrival (the
// producer arrives later, once it has also written the stage's scales).
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ int clamp_len(int L, int Lmax, int *err) {
    if (L < 0 || L > Lmax) {
        set_error(err, GQA_ERR_BAD_PAGE);
        return L < 0 ? 0 : Lmax;
    }
    return L;
}

// Output stores: bf16 (the decode's result) or fp32 (the normalised partial of
// gqa_paged_decode_partial, an input of lse_combine).  idx counts elements.
__device__ __forceinline__ void store_out1(void *out, int f32, size_t idx, float v) {
    if (f32) reinterpret_cast<float *>(out)[idx] = v;
    else reinterpret_cast<__nv_bfloat16 *>(out)[idx] = __float2bfloat16(v);
}
__device__ __forceinline__ void store_out2(void *out, int f32, size_t idx, float v0, float v1) {
    if (f32) reinterpret_cast<float2 *>(out)[idx / 2] = make_float2(v0, v1);
    else reinterpret_cast<__nv_bfloat162 *>(out)[idx / 2] = __floats2bfloat162_rn(v0, v1);
}

// One consumer warp's attention state for up to 8*NT packed heads of one kv head:
// q fragments, the running max / sum per head, and O^T accumulators.
//   fragment lane (gq = lane / 4, cq = lane % 4) holds heads 8*nt + 2*cq (+1) and, for
//   dim tile dt, dims dim0(dt) and dim1(dt).
template <int D, int NT, bool FP8, int TT>
struct WarpAttn {
    static constexpr int KT = D / 16;
    static constexpr int MT = TT / 16;  // 16-token halves of a tile
    uint32_t qf[NT][KT][2];
    float qmul;  // fp8 path: power-of-two prescale bringing q into f16 range
    float vref;  // fp8 path: o holds O / vref (tile V scales enter P as vsc / vref)
    float o[NT][KT][4];
    float m[NT][2], l[NT][2];  // reference (log2 units) and running sum per head column

    __device__ __forceinline__ static int dim0(int dt, int gq) { return dt * 16 + gq; }
    __device__ __forceinline__ static int dim1(int dt, int gq) { return dt * 16 + gq + 8; }

    __device__ __forceinline__ void reset() {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
            for (int dt = 0; dt < KT; ++dt)
#pragma unroll
                for (int e = 0; e < 4; ++e) o[nt][dt][e] = 0.f;
            m[nt][0] = m[nt][1] = -INFINITY;
            l[nt][0] = l[nt][1] = 0.f;
        }
        vref = 0.f;
    }

    // q rows of the nh packed heads start at q_rows (row stride D).
    __device__ __forceinline__ void load_q(const __nv_bfloat16 *q_rows, int nh, int lane) {
        const int gq = lane >> 2, cq = lane & 3;
        qmul = 1.f;
        if (!FP8) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int hl = nt * 8 + gq;
                const bool ok = hl < nh;
                const uint32_t *qw = reinterpret_cast<const uint32_t *>(q_rows + (size_t)(ok ? hl : 0) * D);
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
                const uint2 *qw = reinterpret_cast<const uint2 *>(q_rows + (size_t)(ok ? hl : 0) * D);
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
            for (int o2 = 16; o2 > 0; o2 >>= 1) amax = fmaxf(amax, __shfl_xor_sync(kFull, amax, o2));
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

    // Fold one TT-token tile (valid tokens first, rows past them ignored) into the state.
    // fp8: ksc[mt] / vsc[mt] are the K / V scales of the tile's 16-token half mt (two
    // pages when a 32-token tile spans two 16-token pages).
    __device__ __forceinline__ void tile(uint8_t *kt, uint8_t *vt, int valid, float scale_log2,
                                         const float (&ksc)[2], const float (&vsc)[2], int lane) {
        using C = Cfg<D, FP8, kRingSplit, TT>;
        const int gq = lane >> 2;
        if (valid < TT) {
            // Rows past the end of the sequence may hold anything (even NaN): zero the V
            // rows so 0-weight tokens contribute exactly 0; K rows are masked below.
            constexpr int kChunksPerRow = C::kRowBytes / 16;
            for (int e = lane; e < (TT - valid) * kChunksPerRow; e += 32) {
                const int r = valid + e / kChunksPerRow, cb = (e % kChunksPerRow) * 16;
                *reinterpret_cast<uint4 *>(vt + swz<TT>(r, cb)) = make_uint4(0u, 0u, 0u, 0u);
            }
            __syncwarp();
        }
        const uint32_t kbase = smem_u32(kt), vbase = smem_u32(vt);

        // ---- scores S^T[token][head] = K q^T, per 16-token half
        float s[MT][NT][4];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) s[mt][nt][0] = s[mt][nt][1] = s[mt][nt][2] = s[mt][nt][3] = 0.f;
        if (!FP8) {
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                const int r = (lane & 7) + ((lane >> 3) & 1) * 8 + 16 * mt;
#pragma unroll
                for (int ks = 0; ks < KT; ++ks) {
                    uint32_t af[4];
                    ldsm_x4(af, kbase + swz<TT>(r, (ks * 16 + (lane >> 4) * 8) * 2));
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) mma_bf16(s[mt][nt], af, qf[nt][ks][0], qf[nt][ks][1]);
                }
            }
        } else {
            // the even and odd k steps accumulate in two chains, added at the end: half the
            // dependent MMA latency per 16-token half
            float s2[MT][NT][4];
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) s2[mt][nt][0] = s2[mt][nt][1] = s2[mt][nt][2] = s2[mt][nt][3] = 0.f;
            // One ldmatrix.x4 over 32 fp8 dims serves two k steps; the k order inside a
            // step is permuted identically for K (here) and q (qf), which leaves each dot
            // product unchanged.
            const int j = lane >> 3;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                const int r = (lane & 7) + (j & 1) * 8 + 16 * mt;
#pragma unroll
                for (int kp = 0; kp < D / 32; ++kp) {
                    uint32_t raw[4];
                    ldsm_x4(raw, kbase + swz<TT>(r, 32 * kp + (j >> 1) * 16));
                    uint32_t a0[4], a1[4];
                    e4m3x4_to_f16x4(raw[0], a0[0], a0[2]);
                    e4m3x4_to_f16x4(raw[1], a0[1], a0[3]);
                    e4m3x4_to_f16x4(raw[2], a1[0], a1[2]);
                    e4m3x4_to_f16x4(raw[3], a1[1], a1[3]);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        mma_f16(s[mt][nt], a0, qf[nt][2 * kp][0], qf[nt][2 * kp][1]);
                        mma_f16(s2[mt][nt], a1, qf[nt][2 * kp + 1][0], qf[nt][2 * kp + 1][1]);
                    }
                }
            }
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) s[mt][nt][e] += s2[mt][nt][e];
        }

        // ---- online softmax (exp2 domain) over the tile, per packed head column, with a
        // lazily moved reference: m only moves when a score passes it by more than 2^8
        // (so P <= 2^8), which needs the column max (3 shuffles) and an O rescale only on
        // those rare tiles; every other tile is one vote.
        float kmul[MT];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) kmul[mt] = FP8 ? scale_log2 * ksc[mt] / qmul : scale_log2;
        float x[MT][NT][4];
        bool need = false;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                x[mt][nt][0] = (16 * mt + gq < valid) ? s[mt][nt][0] * kmul[mt] : -INFINITY;
                x[mt][nt][1] = (16 * mt + gq < valid) ? s[mt][nt][1] * kmul[mt] : -INFINITY;
                x[mt][nt][2] = (16 * mt + gq + 8 < valid) ? s[mt][nt][2] * kmul[mt] : -INFINITY;
                x[mt][nt][3] = (16 * mt + gq + 8 < valid) ? s[mt][nt][3] * kmul[mt] : -INFINITY;
                need |= fmaxf(x[mt][nt][0], x[mt][nt][2]) > m[nt][0] + kLazyRef;
                need |= fmaxf(x[mt][nt][1], x[mt][nt][3]) > m[nt][1] + kLazyRef;
            }
        if (__any_sync(kFull, need)) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                float alpha[2];
#pragma unroll
                for (int jj = 0; jj < 2; ++jj) {
                    float mx = -INFINITY;
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt) mx = fmaxf(mx, fmaxf(x[mt][nt][jj], x[mt][nt][jj + 2]));
                    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 4));
                    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 8));
                    mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 16));
                    const float mnew = fmaxf(m[nt][jj], mx);
                    alpha[jj] = fast_exp2(m[nt][jj] - (mnew == -INFINITY ? 0.f : mnew));
                    l[nt][jj] *= alpha[jj];
                    m[nt][jj] = mnew;
                }
#pragma unroll
                for (int dt = 0; dt < KT; ++dt) {
                    o[nt][dt][0] *= alpha[0];
                    o[nt][dt][1] *= alpha[1];
                    o[nt][dt][2] *= alpha[0];
                    o[nt][dt][3] *= alpha[1];
                }
            }
        }
        // fp8: P enters the P.V product as P * vsc / vref, so the MMAs accumulate straight
        // into o; vref follows the tile's larger V scale when the ratio leaves [2^-8, 2^7]
        // (keeping the f16 P under 2^15) and stays put for all-zero pages (vsc = 0).
        float f[MT];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) f[mt] = 1.f;
        if (FP8) {
            const float vmax = MT == 2 ? fmaxf(vsc[0], vsc[1]) : vsc[0];
            if (vref == 0.f) vref = vmax > 0.f ? vmax : 1.f;
            const float fm = vmax / vref;
            if (fm > 128.f || (fm > 0.f && fm < 1.f / 256.f)) {
                const float r = vref / vmax;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int dt = 0; dt < KT; ++dt)
#pragma unroll
                        for (int e = 0; e < 4; ++e) o[nt][dt][e] *= r;
                vref = vmax;
            }
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) f[mt] = vsc[mt] / vref;
        }
        uint32_t pb[MT][NT][2], pbl[MT][NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const float mr0 = m[nt][0] == -INFINITY ? 0.f : m[nt][0];
            const float mr1 = m[nt][1] == -INFINITY ? 0.f : m[nt][1];
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                const float p0 = fast_exp2(x[mt][nt][0] - mr0), p1 = fast_exp2(x[mt][nt][1] - mr1);
                const float p2 = fast_exp2(x[mt][nt][2] - mr0), p3 = fast_exp2(x[mt][nt][3] - mr1);
                l[nt][0] += p0 + p2;
                l[nt][1] += p1 + p3;
                if (!FP8) {
                    // P as a bf16 value plus its bf16 residual: O += V^T P_hi^T + V^T P_lo^T
                    // keeps the weights at ~16 bits (one bf16 P costs up to 2^-9 per weight).
                    uint32_t h0, l0, h1, l1;
                    split_bf16x2(p0, p1, h0, l0);
                    split_bf16x2(p2, p3, h1, l1);
                    pb[mt][nt][0] = movmatrix_trans(h0);
                    pb[mt][nt][1] = movmatrix_trans(h1);
                    pbl[mt][nt][0] = movmatrix_trans(l0);
                    pbl[mt][nt][1] = movmatrix_trans(l1);
                } else {
                    pb[mt][nt][0] = movmatrix_trans(pack_f16(p0 * f[mt], p1 * f[mt]));
                    pb[mt][nt][1] = movmatrix_trans(pack_f16(p2 * f[mt], p3 * f[mt]));
                }
            }
        }

        // ---- O^T[dim][head] += V^T P^T
        if (!FP8) {
            const int j = lane >> 3;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                const int r = (lane & 7) + (j >> 1) * 8 + 16 * mt;
#pragma unroll
                for (int dt = 0; dt < KT; ++dt) {
                    uint32_t af[4];
                    ldsm_x4_trans(af, vbase + swz<TT>(r, (dt * 16 + (j & 1) * 8) * 2));
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        mma_bf16(o[nt][dt], af, pb[mt][nt][0], pb[mt][nt][1]);
                        mma_bf16(o[nt][dt], af, pbl[mt][nt][0], pbl[mt][nt][1]);
                    }
                }
            }
        } else {
            // fp8 V: a transposing byte ldmatrix per 16 tokens x 16 dims gives each lane
            // four tokens of one dim, already in the A fragment's k order once the rows are
            // fed permuted: matrix row i (lane i < 16 gives its address) is token pi(i) of
            // the 16-token half, pi(4c + k) = 2c + (k & 1) + 8 (k >> 1), so lane (g, c)
            // receives tokens 2c, 2c+1, 2c+8, 2c+9 of dims g and g+8; two conversions make
            // the four f16 pairs, with no transpose through registers.
            const int ii = lane & 15;
            const int tok = 2 * (ii >> 2) + (ii & 1) + 8 * ((ii >> 1) & 1);
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                const int r = tok + 16 * mt;
#pragma unroll
                for (int dt = 0; dt < KT; ++dt) {
                    uint32_t w0, w1;
                    ldsm8_trans_x1(w0, w1, vbase + swz<TT>(r, 16 * dt));
                    uint32_t af[4];
                    e4m3x4_to_f16x4(w0, af[0], af[2]);
                    e4m3x4_to_f16x4(w1, af[1], af[3]);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) mma_f16(o[nt][dt], af, pb[mt][nt][0], pb[mt][nt][1]);
                }
            }
        }
    }

    // Sum the per-lane partial sums l over the 8 lanes sharing a head column.
    __device__ __forceinline__ void finish_l() {
        if (FP8 && vref != 0.f) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int dt = 0; dt < KT; ++dt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) o[nt][dt][e] *= vref;
        }
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
    }
};

// ========================================================================== split schedule
template <int D, int NT, bool FP8, int TT>
__global__ void __launch_bounds__(kThreads, NT == 1 ? 3 : 2)
    decode_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                  const DecodeArgs a, const int heads_per_cta, const int head_chunks) {
    using C = Cfg<D, FP8, kRingSplit, TT>;
    constexpr int kTile = TT;
    constexpr int S = C::kStages;
    constexpr int KT = D / 16;
    extern __shared__ uint8_t smem_raw[];
    using SMT = Smem<D, FP8, kRingSplit, TT>;
    SMT &sm = *reinterpret_cast<SMT *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int split = blockIdx.x;
    const int kvh = blockIdx.y / head_chunks, chunk = blockIdx.y % head_chunks;
    const int b = blockIdx.z;
    const int g = a.Hq / a.Hk;
    const int head_lo = kvh * g + chunk * heads_per_cta;
    const int nh = min(heads_per_cta, g - chunk * heads_per_cta);
    const int P = a.P;
    // Launched with programmatic stream serialization: the CTA may be resident before the
    // previous kernel in the stream has finished, and touches no input, output or
    // workspace byte until it has.  lse_combine behind it may be scheduled from here on.
    grid_dependency_wait();
    grid_dependents_launch();

    // This split's token range [t0, t1), page aligned (contiguous ranges of
    // ceil(np / num_splits) pages).
    const int L = clamp_len(a.seq_lens[b], a.pt_stride * P, threadIdx.x == 0 ? a.err : nullptr);
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
                            sm.kscale[stage][0] = sm.kscale[stage][1] = ks;
                            sm.vscale[stage][0] = sm.vscale[stage][1] = vs;
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
    const int gq = lane >> 2, cq = lane & 3;
    WarpAttn<D, NT, FP8, TT> st;
    st.load_q(reinterpret_cast<const __nv_bfloat16 *>(a.q) + ((size_t)b * a.Hq + head_lo) * D, nh, lane);
    st.reset();
    const float scale_log2 = a.scale * kLog2e;

    bool fail = false;
    for (int it = warp; it < n_tiles; it += kConsumerWarps) {
        const int stage = it % S;
        const bool ok = mbar_wait(&sm.full[stage], (it / S) & 1);
        if (__any_sync(kFull, !ok)) {
            fail = true;
            break;
        }
        const float ksl[2] = {FP8 ? sm.kscale[stage][0] : 1.f, FP8 ? sm.kscale[stage][1] : 1.f};
        const float vsl[2] = {FP8 ? sm.vscale[stage][0] : 1.f, FP8 ? sm.vscale[stage][1] : 1.f};
        st.tile(sm.tiles[stage][0], sm.tiles[stage][1], t1 - (t0 + it * kTile), scale_log2,
                ksl, vsl, lane);
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.empty[stage]);
    }

    // ------------------------------------------------------------------ epilogue
    st.finish_l();
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
            const int d0 = WarpAttn<D, NT, FP8, TT>::dim0(dt, gq), d1 = WarpAttn<D, NT, FP8, TT>::dim1(dt, gq);
            float *w = red_o + (size_t)(warp * HW + h0) * RS;
            w[d0] = st.o[nt][dt][0];
            w[RS + d0] = st.o[nt][dt][1];
            w[d1] = st.o[nt][dt][2];
            w[RS + d1] = st.o[nt][dt][3];
        }
        if (gq == 0) {
            red_m[warp * HW + h0] = st.m[nt][0];
            red_m[warp * HW + h0 + 1] = st.m[nt][1];
            red_l[warp * HW + h0] = st.l[nt][0];
            red_l[warp * HW + h0 + 1] = st.l[nt][1];
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
            store_out2(a.out, a.out_f32, row * D + d, o0 * inv, o1 * inv);
            if (d == 0 && a.lse) a.lse[row] = lse_v;
        } else {
            const size_t prow = (size_t)split * rows_total + row;
            reinterpret_cast<float2 *>(a.o_part)[(prow * D + d) / 2] = make_float2(o0 * inv, o1 * inv);
            if (d == 0) a.lse_part[prow] = lse_v;
        }
    }
}

// ========================================================== balanced persistent schedule
//
// Flat tile space: sequence b owns tiles [U*pre[b], U*pre[b+1]) with pre[] the prefix of
// nt_b = ceil(L_b / 16) and U = Hk * head chunks units per sequence; unit y of sequence
// b owns [U*pre[b] + y*nt_b, ... + nt_b).  With T tiles and NW workers (sk_workers: at most
// one per kMinTilesPerWorker tiles, or per kMinTilesPerWorkerSmall for small launches,
// and a multiple of the unit count where the units merge in the launch), worker W owns [W*T/NW, (W+1)*T/NW) (floor divisions): every worker gets one tile more or
// less than any other.
//
// Each consumer warp is one worker with a private sub-ring of S/4 stages fed by its own
// producer lane (lane w of warp 4), so a warp that pauses (loading the next unit's q,
// merging pieces) never holds up the other warps' streams.

constexpr int kMinTilesPerWorker = 16;  // 16-token tiles; half as many 32-token tiles
// When one worker per kMinTilesPerWorker tiles would leave more than three quarters of the
// workers idle (a few short sequences), one per kMinTilesPerWorkerSmall tiles: such
// streams are latency-bound, so more of them in flight finish sooner.
constexpr int kMinTilesPerWorkerSmall = 4;

// Workers of a launch with T tiles of TT tokens, `workers` consumer warps and `units`
// (sequence, kv head, head chunk) units.  Where the units merge in the launch (fewer than
// kDeferMinWorkersPerUnit workers each), the count is rounded down to a multiple of the
// units if that keeps three quarters of the workers: with units of equal length every
// worker then holds one piece of one unit instead of the end of one and the start of the
// next, so it writes one piece, and each unit merges c pieces that finish together.
// Measured (B=20..64 at ctx 2048, bf16 and e4m3): 3-7% faster, no slower elsewhere.
template <int TT>
__device__ __forceinline__ long long sk_workers(long long T, long long workers, long long units) {
    constexpr long long kMin = kMinTilesPerWorker * 16 / TT;
    const long long nw = T / kMin;
    const long long per = nw * 4 < workers ? kMinTilesPerWorkerSmall : kMin;
    const long long r = min(workers, max(1LL, T / per));
    const long long c = units > 0 ? r / units : 0;
    if (c >= 1 && c < kDeferMinWorkersPerUnit && 4 * c * units >= 3 * r) return c * units;
    return r;
}
// Launches whose units average more than kDeferMinWorkersPerUnit workers each leave their
// pieces to a second kernel (piece_merge_kernel, the DEFER instance), which merges every
// cut unit in parallel; otherwise the last piece of a unit to finish merges all of them in
// the same launch.  The two are separate instances so that the in-launch merge's
// registers do not burden the other's streaming loop.

__device__ __forceinline__ long long sk_start(long long W, long long T, long long NW) {
    return W >= NW ? T : (W * T) / NW;
}
// The worker whose range holds flat tile t: max W with sk_start(W) <= t.
__device__ __forceinline__ long long sk_worker_of(long long t, long long T, long long NW) {
    return ((t + 1) * NW + T - 1) / T - 1;
}

// Position (sequence, unit, tile) of flat tile f, and a step to the next flat tile.
struct FlatPos {
    int b, y, tile, nt;
};

__device__ __forceinline__ FlatPos flat_locate(long long f, const int *pre, int B, int U) {
    int lo = 0, hi = B - 1;  // smallest b with U*pre[b+1] > f
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if ((long long)U * pre[mid + 1] > f) hi = mid; else lo = mid + 1;
    }
    FlatPos p;
    p.b = lo;
    p.nt = pre[lo + 1] - pre[lo];
    const long long local = f - (long long)U * pre[lo];
    p.y = (int)(local / p.nt);
    p.tile = (int)(local % p.nt);
    return p;
}

__device__ __forceinline__ void flat_next(FlatPos &p, const int *pre, int U) {
    if (++p.tile < p.nt) return;
    p.tile = 0;
    if (++p.y < U) return;
    p.y = 0;
    do {
        ++p.b;
        p.nt = pre[p.b + 1] - pre[p.b];
    } while (p.nt == 0);
}

// Merge of every piece of one unit (pieces of workers wfirst..wlast; side 1 for the
// first, side 0 for the rest) by one online log-sum-exp pass.  Lane owns dims
// [DV*lane, DV*lane + DV) of every head; each piece's loads are independent of each
// other.
template <int D, int HW>
__device__ __forceinline__ void merge_pieces(const float *pieces, long long wfirst, long long wlast,
                                          int slot_floats, int hpc, int nh, void *out, int out_f32,
                                          size_t out0, float *lse_rows, int lane) {
    constexpr int DV = D / 32;
    float Mh[HW], Wh[HW], acc[HW][DV];
#pragma unroll
    for (int h = 0; h < HW; ++h) {
        Mh[h] = -INFINITY;
        Wh[h] = 0.f;
#pragma unroll
        for (int v = 0; v < DV; ++v) acc[h][v] = 0.f;
    }
    for (long long W = wfirst; W <= wlast; ++W) {
        const float *ps = pieces + (size_t)(W * 2 + (W == wfirst ? 1 : 0)) * slot_floats;
        float lv[HW], ov[HW][DV];
#pragma unroll
        for (int h = 0; h < HW; ++h) {
            if (h < nh) {
                lv[h] = __ldcg(ps + hpc * D + h);
                if constexpr (DV == 4) {
                    const float4 t = __ldcg(reinterpret_cast<const float4 *>(ps + h * D + DV * lane));
                    ov[h][0] = t.x; ov[h][1] = t.y; ov[h][2] = t.z; ov[h][3] = t.w;
                } else {
                    const float2 t = __ldcg(reinterpret_cast<const float2 *>(ps + h * D + DV * lane));
                    ov[h][0] = t.x; ov[h][1] = t.y;
                }
            }
        }
#pragma unroll
        for (int h = 0; h < HW; ++h) {
            if (h >= nh) continue;
            const float mnew = fmaxf(Mh[h], lv[h]);
            const float c_old = __expf(Mh[h] - mnew), c_new = __expf(lv[h] - mnew);
            Wh[h] = Wh[h] * c_old + c_new;
#pragma unroll
            for (int v = 0; v < DV; ++v) acc[h][v] = acc[h][v] * c_old + c_new * ov[h][v];
            Mh[h] = mnew;
        }
    }
#pragma unroll
    for (int h = 0; h < HW; ++h) {
        if (h >= nh) continue;
        const float inv = 1.f / Wh[h];
        const size_t e0 = out0 + (size_t)h * D + DV * lane;
#pragma unroll
        for (int v = 0; v < DV; v += 2) store_out2(out, out_f32, e0 + v, acc[h][v] * inv, acc[h][v + 1] * inv);
        if (lane == 0 && lse_rows) lse_rows[h] = Mh[h] + logf(Wh[h]);
    }
}

// Tiles per sequence and their exclusive prefix into pre[0..B] (one warp; lane i owns a
// run of sequences).  Lengths are clamped to the page table; err (if not null) records a
// clamped length.
template <int TT>
__device__ __forceinline__ void tile_prefix(const DecodeArgs &a, int *pre, int Lmax, int *err, int lane) {
    const int B = a.B;
    const int per = (B + 31) / 32;
    const int b0 = min(B, lane * per), b1 = min(B, b0 + per);
    int sum = 0;
    for (int b = b0; b < b1; ++b) sum += (clamp_len(a.seq_lens[b], Lmax, err) + TT - 1) / TT;
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += t;
    }
    int run = incl - sum;
    for (int b = b0; b < b1; ++b) {
        pre[b] = run;
        run += (clamp_len(a.seq_lens[b], Lmax, nullptr) + TT - 1) / TT;
    }
    if (lane == 31) pre[B] = incl;
}

template <int D, int NT, bool FP8, int TT, bool DEFER>
__global__ void __launch_bounds__(balanced_threads<FP8>(), kStreamCtasPerSm)
    decode_sk_kernel(const __grid_constant__ CUtensorMap kmap,
                     const __grid_constant__ CUtensorMap vmap, const DecodeArgs a,
                     const int heads_per_cta, const int head_chunks) {
    using C = Cfg<D, FP8, kRingBalanced, TT>;
    using SM = Smem<D, FP8, kRingBalanced, TT>;
    using WA = WarpAttn<D, NT, FP8, TT>;
    constexpr int kTile = TT;
    constexpr int S = C::kStages;
    constexpr int SW = S / kConsumerWarps;  // stages per worker
    constexpr int KT = D / 16;
    constexpr int HW = 8 * NT;               // packed head columns
    extern __shared__ uint8_t smem_raw[];
    SM &sm = *reinterpret_cast<SM *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    int *pre = reinterpret_cast<int *>(reinterpret_cast<uint8_t *>(&sm) + sizeof(SM));

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int B = a.B, P = a.P, g = a.Hq / a.Hk;
    const int U = a.Hk * head_chunks;
    const int Lmax = a.pt_stride * P;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        sm.abort_flag = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == kConsumerWarps && lane == 0) {
        prefetch_tensormap(&kmap);
        prefetch_tensormap(&vmap);
    }
    // Everything above may overlap the previous kernel in the stream; the inputs (and the
    // workspace) are read only after it has completed.
    grid_dependency_wait();
    grid_dependents_launch();
    if (warp == 1) {
        // the page table into L2 while warp 0 waits for seq_lens: 128-byte lines spread
        // over the grid, at most 64 per CTA
        const char *pt0 = reinterpret_cast<const char *>(a.page_table);
        const long long lines = ((long long)B * a.pt_stride * 4 + 127) / 128;
        for (long long i = blockIdx.x + (long long)gridDim.x * lane, k = 0; i < lines && k < 2;
             i += (long long)gridDim.x * 32, ++k)
            prefetch_l2(pt0 + i * 128);
    }

    // Tiles per sequence and their exclusive prefix (warp 0).
    if (warp == 0) tile_prefix<kTile>(a, pre, Lmax, blockIdx.x == 0 ? a.err : nullptr, lane);
    __syncthreads();

    const long long T = (long long)U * pre[B];
    const long long NW = sk_workers<TT>(T, (long long)gridDim.x * kConsumerWarps, (long long)B * U);
    const long long W0cta = (long long)blockIdx.x * kConsumerWarps;

    // Sequences with no tokens have no tiles: their outputs are written here (zeros, -inf).
    for (int b = blockIdx.x; b < B; b += gridDim.x) {
        if (pre[b + 1] != pre[b]) continue;
        for (int e = threadIdx.x; e < a.Hq * D; e += blockDim.x)
            store_out1(a.out, a.out_f32, (size_t)b * a.Hq * D + e, 0.f);
        if (a.lse)
            for (int e = threadIdx.x; e < a.Hq; e += blockDim.x) a.lse[(size_t)b * a.Hq + e] = -INFINITY;
    }
    if (T == 0) return;

    if (warp >= kConsumerWarps) {
        // ---------------------------------------------- producer of worker w: lane w of
        // warp 4 (bf16), or lane 0 of warp 4 + w (e4m3)
        if (FP8) {
            regs_release<kRegsProducer>();
            if (lane != 0) return;
        } else if (lane >= kConsumerWarps) {
            return;
        }
        const int w = FP8 ? warp - kConsumerWarps : lane;
        const uint64_t pol = a.pack_gqa ? policy_evict_first() : policy_evict_last();
        const long long s_w = sk_start(W0cta + w, T, NW), e_w = sk_start(W0cta + w + 1, T, NW);
        const long long n = e_w - s_w;
        long long issued = 0;
        FlatPos pos;
        if (n > 0) pos = flat_locate(s_w, pre, B, U);
        for (long long r = 0; r < n; ++r) {
            if (r > 0) flat_next(pos, pre, U);
            const int stage = w * SW + (int)(r % SW);
            const long long use = r / SW;
            if (use > 0 && !mbar_wait(&sm.empty[stage], (uint32_t)((use - 1) & 1))) {
                set_error(a.err, GQA_ERR_TIMEOUT);
                break;
            }
            const int L = clamp_len(a.seq_lens[pos.b], Lmax, nullptr);
            const int tok0 = pos.tile * kTile;
            const int kvh = pos.y / head_chunks;
            TileRec rec;
            rec.b = pos.b;
            rec.y = pos.y;
            rec.tile = pos.tile;
            rec.valid = min(kTile, L - tok0);
            rec.f = s_w + r;
            // a 32-token e4m3 tile on 16-token pages spans two pages: one box from each
            const int32_t *ptb = a.page_table + (size_t)pos.b * a.pt_stride + tok0 / P;
            const int phys = __ldg(ptb);
            const bool two = kTile > P;
            const bool second = two && tok0 + P < L;
            const int phys2 = second ? __ldg(ptb + 1) : phys;
            sm.rec[stage] = rec;
            if (phys < 0 || phys >= a.num_pages || phys2 < 0 || phys2 >= a.num_pages) {
                set_error(a.err, GQA_ERR_BAD_PAGE);
                mbar_arrive(&sm.full[stage]);  // no copy: the tile computes on stale data
            } else {
                // e4m3: the copies are issued first (expected bytes, no arrival), the scales are
                // loaded while they fly, and the producer's arrival after the scales' stores
                // releases both.  Loading the scales first put a second dependent round trip
                // (page-table entry, then scales) before every copy.
                const int row = (phys * a.Hk + kvh) * P + tok0 % P;
                if (!two) {
                    if (FP8) mbar_expect_tx(&sm.full[stage], 2 * C::kTileBytes);
                    else mbar_arrive_expect_tx(&sm.full[stage], 2 * C::kTileBytes);
#pragma unroll
                    for (int bx = 0; bx < C::kBoxes; ++bx) {
                        tma_load_2d(sm.tiles[stage][0] + bx * kTile * 128, &kmap, &sm.full[stage],
                                    bx * C::kBoxCols, row, pol);
                        tma_load_2d(sm.tiles[stage][1] + bx * kTile * 128, &vmap, &sm.full[stage],
                                    bx * C::kBoxCols, row, pol);
                    }
                } else {
                    // P-row boxes; rows past the first page are the second page's
                    const int row2 = (phys2 * a.Hk + kvh) * P;
                    if (FP8) mbar_expect_tx(&sm.full[stage], (second ? 2 : 1) * 2 * C::kBoxes * P * 128);
                    else mbar_arrive_expect_tx(&sm.full[stage], (second ? 2 : 1) * 2 * C::kBoxes * P * 128);
#pragma unroll
                    for (int bx = 0; bx < C::kBoxes; ++bx) {
                        tma_load_2d(sm.tiles[stage][0] + bx * kTile * 128, &kmap, &sm.full[stage],
                                    bx * C::kBoxCols, row, pol);
                        tma_load_2d(sm.tiles[stage][1] + bx * kTile * 128, &vmap, &sm.full[stage],
                                    bx * C::kBoxCols, row, pol);
                        if (second) {
                            tma_load_2d(sm.tiles[stage][0] + bx * kTile * 128 + P * 128, &kmap,
                                        &sm.full[stage], bx * C::kBoxCols, row2, pol);
                            tma_load_2d(sm.tiles[stage][1] + bx * kTile * 128 + P * 128, &vmap,
                                        &sm.full[stage], bx * C::kBoxCols, row2, pol);
                        }
                    }
                }
                if (FP8) {
                    sm.kscale[stage][0] = __ldg(a.k_scale + (size_t)phys * a.Hk + kvh);
                    sm.vscale[stage][0] = __ldg(a.v_scale + (size_t)phys * a.Hk + kvh);
                    sm.kscale[stage][1] = second ? __ldg(a.k_scale + (size_t)phys2 * a.Hk + kvh) : sm.kscale[stage][0];
                    sm.vscale[stage][1] = second ? __ldg(a.v_scale + (size_t)phys2 * a.Hk + kvh) : sm.vscale[stage][0];
                    mbar_arrive(&sm.full[stage]);
                }
            }
            issued = r + 1;
        }
        // no copy into this CTA's shared memory may outlive it
        for (long long r = max(0LL, issued - SW); r < issued; ++r)
            if (!mbar_wait(&sm.full[w * SW + (int)(r % SW)], (uint32_t)((r / SW) & 1))) {
                set_error(a.err, GQA_ERR_TIMEOUT);
                break;
            }
        return;
    }

    // -------------------------------------------------------------------- consumers
    if (FP8) regs_acquire<kRegsConsumer>();
    const int gq = lane >> 2, cq = lane & 3;
    const long long Wme = W0cta + warp;
    const long long s_w = sk_start(Wme, T, NW), e_w = sk_start(Wme + 1, T, NW);
    const long long n = e_w - s_w;
    const float scale_log2 = a.scale * kLog2e;
    // piece slot: heads_per_cta rows of D, then heads_per_cta lse values, padded to a
    // multiple of 4 floats so every slot (and row) starts 16-byte aligned for the merge
    const int slot_floats = (heads_per_cta * (D + 1) + 3) & ~3;
    WA st;
    st.reset();
    st.qmul = 1.f;
    int cur_b = -1, cur_y = -1;
    if (n > 0) {
        // the first unit's q is loaded while the producer resolves and copies the first tile
        const FlatPos p0 = flat_locate(s_w, pre, B, U);
        const int kvh = p0.y / head_chunks, chunk = p0.y % head_chunks;
        st.load_q(reinterpret_cast<const __nv_bfloat16 *>(a.q) +
                      ((size_t)p0.b * a.Hq + kvh * g + chunk * heads_per_cta) * D,
                  min(heads_per_cta, g - chunk * heads_per_cta), lane);
        cur_b = p0.b;
        cur_y = p0.y;
    }
    for (long long r = 0; r < n; ++r) {
        const int stage = warp * SW + (int)(r % SW);
        const bool ok = mbar_wait(&sm.full[stage], (uint32_t)((r / SW) & 1));
        if (__any_sync(kFull, !ok)) {
            if (lane == 0) set_error(a.err, GQA_ERR_TIMEOUT);
            break;
        }
        const TileRec rec = sm.rec[stage];
        const float ks[2] = {FP8 ? sm.kscale[stage][0] : 1.f, FP8 ? sm.kscale[stage][1] : 1.f};
        const float vs[2] = {FP8 ? sm.vscale[stage][0] : 1.f, FP8 ? sm.vscale[stage][1] : 1.f};
        const int b = rec.b, y = rec.y;
        const int kvh = y / head_chunks, chunk = y % head_chunks;
        const int head_lo = kvh * g + chunk * heads_per_cta;
        const int nh = min(heads_per_cta, g - chunk * heads_per_cta);
        if (b != cur_b || y != cur_y) {
            st.reset();
            st.load_q(reinterpret_cast<const __nv_bfloat16 *>(a.q) + ((size_t)b * a.Hq + head_lo) * D,
                      nh, lane);
            cur_b = b;
            cur_y = y;
        }
        st.tile(sm.tiles[stage][0], sm.tiles[stage][1], rec.valid, scale_log2, ks, vs, lane);
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.empty[stage]);
        const int nt_b = pre[b + 1] - pre[b];
        if (rec.tile != nt_b - 1 && rec.f != e_w - 1) continue;

        // ---- this warp's share of unit (b, y) is done
        st.finish_l();
        const long long us = (long long)U * pre[b] + (long long)y * nt_b, ue = us + nt_b;
        const size_t row0 = (size_t)b * a.Hq + head_lo;
        if (us >= s_w && ue <= e_w) {
            // the whole unit: write the output directly
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int jj = 0; jj < 2; ++jj) {
                    const int h = nt * 8 + 2 * cq + jj;
                    if (h >= nh) continue;
                    const float inv = st.l[nt][jj] > 0.f ? 1.f / st.l[nt][jj] : 0.f;
                    const size_t e0 = (row0 + h) * D;
#pragma unroll
                    for (int dt = 0; dt < KT; ++dt) {
                        store_out1(a.out, a.out_f32, e0 + WA::dim0(dt, gq), st.o[nt][dt][jj] * inv);
                        store_out1(a.out, a.out_f32, e0 + WA::dim1(dt, gq), st.o[nt][dt][jj + 2] * inv);
                    }
                    if (gq == 0 && a.lse)
                        a.lse[row0 + h] = st.l[nt][jj] > 0.f
                                              ? (st.m[nt][jj] + __log2f(st.l[nt][jj])) * kLn2
                                              : -INFINITY;
                }
        } else {
            // A piece of a unit shared with neighbouring workers: side 0 = the unit began
            // before this worker's range, side 1 = it begins here and continues after.
            // The piece is written normalised, with its natural-log LSE.  Launches whose
            // units span few workers: the last piece to finish merges all of them in one
            // pass.  Launches whose units span many (DEFER): piece_merge_kernel merges
            // them after this launch.
            const long long wfirst = sk_worker_of(us, T, NW), wlast = sk_worker_of(ue - 1, T, NW);
            const int np = (int)(wlast - wfirst + 1);
            const int side = us < s_w ? 0 : 1;
            float *slot = a.pieces + (size_t)(Wme * 2 + side) * slot_floats;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int jj = 0; jj < 2; ++jj) {
                    const int h = nt * 8 + 2 * cq + jj;
                    if (h >= nh) continue;
                    const float inv = 1.f / st.l[nt][jj];
#pragma unroll
                    for (int dt = 0; dt < KT; ++dt) {
                        slot[h * D + WA::dim0(dt, gq)] = st.o[nt][dt][jj] * inv;
                        slot[h * D + WA::dim1(dt, gq)] = st.o[nt][dt][jj + 2] * inv;
                    }
                    if (gq == 0) slot[heads_per_cta * D + h] = (st.m[nt][jj] + __log2f(st.l[nt][jj])) * kLn2;
                }
            if (!DEFER) {
                __threadfence();
                __syncwarp();
                int *ctr = a.counters + (size_t)b * U + y;
                int last = 0;
                if (lane == 0) last = atomicAdd(ctr, 1) == np - 1;
                last = __shfl_sync(kFull, last, 0);
                if (last) {
                    __threadfence();
                    merge_pieces<D, HW>(a.pieces, wfirst, wlast, slot_floats, heads_per_cta, nh,
                                        a.out, a.out_f32, row0 * D, a.lse ? a.lse + row0 : nullptr,
                                        lane);
                    if (lane == 0) *ctr = 0;  // ready for the next launch
                }
            }
        }
        st.reset();
        cur_b = -1;
    }
}

// Merge of the pieces a DEFER launch of decode_sk_kernel left: one CTA per (unit, head)
// of a cut unit.  It recomputes the launch's partition (the same tile prefix, worker count
// and owners), skips units that one worker held whole, and merges pieces wfirst..wlast by
// log-sum-exp (the merge of NumSplits partials, "解锁GQA性能潜力：从批量大小敏感性到高效优化实践",
// PackGQA / NumSplits section): the pieces' LSEs go to shared memory in one round of
// loads; every warp finds M = max lse and W = sum exp(lse - M) there; warp w sums
// exp(lse_k - M) o_k over pieces k = w, w + 8, ..., eight loads in flight; the eight
// partial sums are added in warp order.  The result does not depend on which worker
// finished first.
constexpr int kMergeWarps = 8;

template <int D, int TT>
__global__ void __launch_bounds__(32 * kMergeWarps)
    piece_merge_kernel(const DecodeArgs a, const int heads_per_cta, const int head_chunks) {
    constexpr int DV = D / 32;
    __shared__ float part[kMergeWarps][D];
    __shared__ float lse_s[kStreamMaxWorkers];  // a unit has at most one piece per worker
    extern __shared__ int pre_m[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int U = a.Hk * head_chunks;
    const int g = a.Hq / a.Hk;
    const int h = blockIdx.y;
    // the pieces are written by the previous kernel in the stream
    grid_dependency_wait();
    if (warp == 0) tile_prefix<TT>(a, pre_m, a.pt_stride * a.P, nullptr, lane);
    __syncthreads();
    const long long T = (long long)U * pre_m[a.B];
    const long long NW = sk_workers<TT>(T, (long long)a.grid * kConsumerWarps, (long long)a.B * U);
    const int slot_floats = (heads_per_cta * (D + 1) + 3) & ~3;
    for (long long u = blockIdx.x; u < (long long)a.B * U; u += gridDim.x) {
        const int b = (int)(u / U), y = (int)(u % U);
        const int nt_b = pre_m[b + 1] - pre_m[b];
        const int kvh = y / head_chunks, chunk = y % head_chunks;
        const int nh = min(heads_per_cta, g - chunk * heads_per_cta);
        if (nt_b == 0 || h >= nh) continue;  // uniform for the CTA
        const long long us = (long long)U * pre_m[b] + (long long)y * nt_b, ue = us + nt_b;
        const long long wfirst = sk_worker_of(us, T, NW), wlast = sk_worker_of(ue - 1, T, NW);
        if (wfirst == wlast) continue;  // written whole by its worker
        const int np = (int)(wlast - wfirst + 1);
        auto slot = [&](int k) -> const float * {
            const long long w = wfirst + k;
            return a.pieces + (size_t)(w * 2 + (k == 0 ? 1 : 0)) * slot_floats;
        };
        // every piece's LSE into shared memory, then M and W (each warp, from there)
        for (int k = threadIdx.x; k < np; k += blockDim.x) lse_s[k] = __ldcg(slot(k) + heads_per_cta * D + h);
        __syncthreads();
        float M = -INFINITY;
        for (int k = lane; k < np; k += 32) M = fmaxf(M, lse_s[k]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(kFull, M, o));
        float W = 0.f;
        for (int k = lane; k < np; k += 32) W += __expf(lse_s[k] - M);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) W += __shfl_xor_sync(kFull, W, o);
        // this warp's pieces
        float acc[DV];
#pragma unroll
        for (int v = 0; v < DV; ++v) acc[v] = 0.f;
#pragma unroll 8
        for (int k = warp; k < np; k += kMergeWarps) {
            const float *ps = slot(k);
            const float wk = __expf(lse_s[k] - M);
            if constexpr (DV == 4) {
                const float4 t = __ldcg(reinterpret_cast<const float4 *>(ps + h * D + DV * lane));
                acc[0] += wk * t.x; acc[1] += wk * t.y; acc[2] += wk * t.z; acc[3] += wk * t.w;
            } else {
                const float2 t = __ldcg(reinterpret_cast<const float2 *>(ps + h * D + DV * lane));
                acc[0] += wk * t.x; acc[1] += wk * t.y;
            }
        }
#pragma unroll
        for (int v = 0; v < DV; ++v) part[warp][DV * lane + v] = acc[v];
        __syncthreads();
        const int head_lo = kvh * g + chunk * heads_per_cta;
        const float inv = 1.f / W;
        for (int d = threadIdx.x; d < D; d += blockDim.x) {
            float sum = 0.f;
#pragma unroll
            for (int w = 0; w < kMergeWarps; ++w) sum += part[w][d];
            store_out1(a.out, a.out_f32, ((size_t)b * a.Hq + head_lo + h) * D + d, sum * inv);
        }
        if (threadIdx.x == 0 && a.lse) a.lse[(size_t)b * a.Hq + head_lo + h] = M + logf(W);
        __syncthreads();  // part[] and lse_s[] are reused by the next unit
    }
}

template <int D, int NT, bool FP8, int TT>
cudaError_t launch_t(const DecodeArgs &a, const CUtensorMap &kmap, const CUtensorMap &vmap,
                     cudaStream_t stream) {
    static_assert(sizeof(float) * kConsumerWarps * 8 * NT * (D + 6) <=
                      sizeof(uint8_t) * Cfg<D, FP8, kRingSplit, TT>::kStages * 2 *
                          Cfg<D, FP8, kRingSplit, TT>::kTileBytes,
                  "reduction area must fit in the stage ring");
    const int g = a.Hq / a.Hk;
    const int hpc = a.pack_gqa ? (g < 8 * NT ? g : 8 * NT) : 1;
    const int chunks = (g + hpc - 1) / hpc;
    if (a.stream_k) {
        const size_t smem =
            sizeof(Smem<D, FP8, kRingBalanced, TT>) + 1024 + sizeof(int) * (size_t)(a.B + 1);
        const bool defer = decode_defers_merge(a.B, a.Hq, a.Hk, a.pack_gqa, a.grid);
        // the 16-head instance (NT = 2) always defers (decode_defers_merge): it has no
        // in-launch-merge instance
        auto kern = defer ? decode_sk_kernel<D, NT, FP8, TT, true> : decode_sk_kernel<D, NT, FP8, TT, NT == 2>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        // programmatic stream serialization: the kernel's set-up overlaps the tail of the
        // previous kernel in the stream (the kernel waits for it before reading inputs)
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(a.grid);
        cfg.blockDim = dim3(balanced_threads<FP8>());
        cfg.dynamicSmemBytes = smem;
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = cudaLaunchKernelEx(&cfg, kern, kmap, vmap, a, hpc, chunks);
        if (e != cudaSuccess || !defer) return e;
        // the merge of the cut units: an ordinary launch (measured faster than letting its
        // CTAs wait beside the decode kernel's)
        const long long nunits = (long long)a.B * a.Hk * chunks;
        piece_merge_kernel<D, TT><<<dim3((unsigned)(nunits < 4096 ? nunits : 4096), (unsigned)hpc),
                                    32 * kMergeWarps, sizeof(int) * (size_t)(a.B + 1), stream>>>(
            a, hpc, chunks);
        return cudaGetLastError();
    }
    const size_t smem = sizeof(Smem<D, FP8, kRingSplit, TT>) + 1024;
    cudaError_t e = cudaFuncSetAttribute(decode_kernel<D, NT, FP8, TT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.num_splits, a.Hk * chunks, a.B);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_kernel<D, NT, FP8, TT>, kmap, vmap, a, hpc, chunks);
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs &a, const CUtensorMap &kmap, const CUtensorMap &vmap,
                          cudaStream_t stream) {
    const int g = a.Hq / a.Hk;
    const bool wide = a.pack_gqa && g > 8;
    if (a.kv_dtype == GQA_KV_FP8_E4M3) {
        // 32-token tiles: the balanced schedule on any page size (two boxes on 16-token
        // pages), the split schedule where a page holds a whole tile
        if (a.stream_k || decode_tile_tokens(a.kv_dtype, a.P) == 32)
            return wide ? launch_t<128, 2, true, 32>(a, kmap, vmap, stream)
                        : launch_t<128, 1, true, 32>(a, kmap, vmap, stream);
        return wide ? launch_t<128, 2, true, 16>(a, kmap, vmap, stream)
                    : launch_t<128, 1, true, 16>(a, kmap, vmap, stream);
    }
    if (a.D == 128)
        return wide ? launch_t<128, 2, false, 16>(a, kmap, vmap, stream)
                    : launch_t<128, 1, false, 16>(a, kmap, vmap, stream);
    return wide ? launch_t<64, 2, false, 16>(a, kmap, vmap, stream)
                : launch_t<64, 1, false, 16>(a, kmap, vmap, stream);
}

}  // namespace gqa
