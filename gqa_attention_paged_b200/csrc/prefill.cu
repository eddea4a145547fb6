// prefill.cu -- causal chunked prefill over a paged KV cache on sm_100a tensor cores.
//
// A chunk of Lq new query tokens per sequence is appended after a paged prior context
// ("TensorRT对Grouped Query Attention的支持进展", section "与动态批处理协同": chunked
// prefill); its K/V are already the last Lq cached tokens, and query row i (position
// L - Lq + i) attends to keys 0 .. L - Lq + i.
//
// One CTA = (two query tiles, kv head, sequence), launched longest first (a one-CTA plan
// kernel orders the work items by the KV tiles they read, before each prefill launch).  A tile packs the g query heads of the
// group with T = 128 / g tokens into 128 rows, row r = (token r / g, head r % g)
// (PackGQA: "解锁GQA性能潜力：从批量大小敏感性到高效优化实践", PackGQA / NumSplits
// section), so each K/V tile feeds every head of the group, twice (once per query tile).
// The attention is the tiled fused form ("TensorRT-LLM与TensorRT核心差异解析", section
// 4.2.1): per 128-key tile, S = Q K^T on tcgen05 into tensor memory, an fp32 online
// softmax in registers, P written back into tensor memory over S, and O += P V on
// tcgen05 with P read from tensor memory.
//
// Warp roles (384 threads, three warpgroups):
//   warp 0      TMA producer: both Q tiles (3-D map over [total_q][Hq][D]), then the K
//               tiles, 16 keys per copy, gathered page by page through the page table.
//   warp 1      allocates all 512 tensor-memory columns (S0, S1, O0, O1) and issues the
//               MMAs from one thread in the order PV0(j), S0(j+1), PV1(j), S1(j+1), so the
//               tensor core works on one query tile while the other one's softmax runs.
//   warps 2-3   load the V tiles (warp 2, the same way) and convert each in place from
//               bf16 to f16, keys past the sequence zeroed first; a tile with a value
//               beyond the f16 range is copied again and stays bf16.
//   warps 4-7   softmax of query tile 0, warps 8-11 of query tile 1; a thread owns one
//               row (one tensor-memory lane) and holds its 128 scores in registers.
// The softmax warpgroups take most of the register file (setmaxnreg).
//
// P precision: P is written as f16 (11 significant bits) and multiplied with the f16
// copy of V, so O += P V keeps each weight to 2^-12 relative.  A V tile holding a value
// of magnitude 2^16 or more (or Inf / NaN) stays bf16; for that tile P is written as a
// bf16 value plus its bf16 residual and O += P_hi V + P_lo V (~16 significant bits).
// The running max is only moved when a row's max grows by more than 2^8, so O is
// rescaled rarely and P stays below 2^8; the final O / l is exact for any reference.
// Every wait is bounded; on expiry the kernel records GQA_ERR_TIMEOUT, finishes its
// outstanding copies and MMAs (bounded), frees its tensor memory and returns.
#include "gqa_device.cuh"
#include "gqa_internal.h"

namespace gqa {
namespace {

constexpr int kM = 128;                // packed query rows per query tile
constexpr int kQT = 2;                 // query tiles per CTA
constexpr int kN = 128;                // keys per KV tile
constexpr int kKStages = 2;            // K ring depth
constexpr int kVStages = 3;            // V ring depth (a V tile also waits for its conversion)
constexpr int kThreadsP = 384;
constexpr int kHalfBytes = kM * 128;   // one 64-column (128-byte) half of a 128-row tile
// A 128-row tile of head dim D: D / 64 halves.
template <int D>
__host__ __device__ constexpr int tile_bytes() { return (D / 64) * kHalfBytes; }
constexpr int kChunk = 16;             // keys per TMA copy (one box)
constexpr int kChunkBytes = kChunk * 128;
constexpr float kLog2eP = 1.4426950408889634f;
constexpr float kLn2P = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
constexpr unsigned kAll = 0xffffffffu;
// Register split: warpgroup 0 (producer, MMA, converters) keeps 64 per thread, the two
// softmax warpgroups take 216: 128*64 + 256*216 <= 384*168, the launch allocation.
constexpr int kRegsSide = 64;
constexpr int kRegsSoftmax = 216;
static_assert(128 * kRegsSide + 256 * kRegsSoftmax <= kThreadsP * 168, "register split");
constexpr int kConvThreads = 64;

template <int D>
struct alignas(1024) PSmem {
    uint8_t q[kQT][tile_bytes<D>()];
    uint8_t k[kKStages][tile_bytes<D>()];
    uint8_t v[kVStages][tile_bytes<D>()];
    uint64_t q_full;
    uint64_t k_full[kKStages], k_empty[kKStages];
    uint64_t v_full[kVStages], v_ready[kVStages], v_empty[kVStages];
    uint64_t s_full[kQT], p_full[kQT], pv_done[kQT];
    uint64_t mma_done;
    uint64_t v_fixsync, v_fix;  // a V tile out of f16 range: both converters done, copied again
    int v_bf16[kVStages];       // 1: the V tile stayed bf16 (a value out of f16 range)
    int conv_ovf[kVStages][2];  // per converter warp: (tile + 1) * 2 + out-of-range flag
    uint32_t tmem_base;
};

static_assert(sizeof(PSmem<128>) + 1024 <= 227 * 1024, "shared memory per CTA");

__device__ __forceinline__ bool wait_all(uint64_t *bar, uint32_t parity) {
    const bool ok = mbar_wait(bar, parity);
    return !__any_sync(kAll, !ok);
}

// KV row (in the [num_pages*Hk*P][D] view) of the 16-key chunk `lane` of KV tile j, or -1
// for lanes past the 8 chunks, keys at or past L, and out-of-range page entries (which
// set GQA_ERR_BAD_PAGE).
__device__ __forceinline__ int kv_chunk_row(const PrefillArgs &a, const int32_t *pt, int j,
                                            int lane, int kvh, int L) {
    const int key0 = j * kN + kChunk * lane;
    if (lane >= kN / kChunk || key0 >= L) return -1;
    const int phys = __ldg(pt + key0 / a.P);
    if (phys < 0 || phys >= a.num_pages) {
        set_error(a.err, GQA_ERR_BAD_PAGE);
        return -1;
    }
    return (phys * a.Hk + kvh) * a.P + key0 % a.P;
}

// Softmax warpgroup of query tile (warp - 4) / 4: online softmax over the score tiles in
// tensor memory, P written back over S, final O / l and LSE to global memory.
template <int D>
__device__ __forceinline__ void softmax_role(PSmem<D> &sm, const PrefillArgs &a, const uint32_t tmem,
                                             const int warp, const int lane, const int (&n_kv_q)[kQT],
                                             const int b, const int kvh, const int g, const int q0,
                                             const int Lq, const int i0, const int T, const int L) {
    // ------------------------------------------------------------ softmax warpgroups
    const int q = (warp - 4) / 4;  // query tile
    const int quad = warp & 3;     // tensor-memory lane quadrant this warp may access
    const int row = quad * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
    const uint32_t tS = tmem + 128 * q + lane_off, tO = tmem + 256 + 128 * q + lane_off;
    const int nk = n_kv_q[q];
    const int ntok = min(T, Lq - (i0 + q * T));
    const bool valid_row = row < ntok * g;
    const int tok = i0 + q * T + row / g;
    const int hh = row % g;
    const int lim = a.causal ? min(L - Lq + tok, L - 1) : L - 1;  // last visible key
    const float c = a.scale * kLog2eP;
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nk; ++j) {
        const int stage = j % kVStages;
        if (!wait_all(&sm.s_full[q], j & 1)) {
            ok = false;
            break;
        }
        tc_fence_after_sync();
        // the row's 128 scores: all four loads in flight before one wait
        uint32_t sr[4][32];
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) tmem_ld32(tS + 32 * cc, sr[cc]);
        tmem_wait_ld();
        const int nvis = lim - j * kN + 1;  // keys of this tile the row may see
        if (nvis < kN) {  // diagonal / tail tile: scores past nvis -> -inf
#pragma unroll
            for (int cc = 0; cc < 4; ++cc)
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    if (32 * cc + e >= nvis) sr[cc][e] = __float_as_uint(-INFINITY);
        }
        float mx;
        {
            float m4[4];
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                float t = fmax3(__uint_as_float(sr[cc][0]), __uint_as_float(sr[cc][1]),
                                __uint_as_float(sr[cc][2]));
#pragma unroll
                for (int e = 3; e < 31; e += 2)
                    t = fmax3(t, __uint_as_float(sr[cc][e]), __uint_as_float(sr[cc][e + 1]));
                m4[cc] = fmaxf(t, __uint_as_float(sr[cc][31]));
            }
            mx = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3]));
        }
        mx *= c;  // c > 0: the max commutes with the scale
        const bool need = mx > m_ref + kRescaleThreshold;
        const float new_ref = need ? mx : m_ref;
        const float mref0 = new_ref == -INFINITY ? 0.f : new_ref;
        const float alpha = ex2_approx(m_ref - mref0);

        if (j > 0 && __any_sync(kAll, need)) {
            // O must not be touched while PV(j-1) still accumulates into it
            if (!wait_all(&sm.pv_done[q], (j - 1) & 1)) {
                ok = false;
                break;
            }
            tc_fence_after_sync();
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t o[32];
                tmem_ld32(tO + 32 * cc, o);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                tmem_st32(tO + 32 * cc, o);
            }
        }
        // P = 2^(s*c - ref) as f16 value pairs, computed while V tile j may still be
        // converting (almost every tile becomes f16); the keys of chunk cc go to columns
        // [32cc, 32cc+16) of S.  Keys go in pairs through the paired fp32 instructions.
        const unsigned long long c2 = f2_pack(c, c), nref2 = f2_pack(-mref0, -mref0);
        unsigned long long sum2 = 0ull;  // (0.f, 0.f)
        uint32_t pk[4][16];
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                float x0, x1;
                f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[cc][2 * e]),
                                         __uint_as_float(sr[cc][2 * e + 1])),
                                 c2, nref2),
                          x0, x1);
                const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
                sum2 = f2_add(sum2, f2_pack(p0, p1));
                pk[cc][e] = pack_f16(p0, p1);
            }
        }
        if (!wait_all(&sm.v_ready[stage], (j / kVStages) & 1)) {
            ok = false;
            break;
        }
        const bool vbf = sm.v_bf16[stage] != 0;
        if (!vbf) {
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) tmem_st16(tS + 32 * cc, pk[cc]);
        } else {
            // the tile stayed bf16: P again from S (not yet overwritten), as bf16 value
            // pairs in [32cc, 32cc+16) and their bf16 residuals in [32cc+16, 32cc+32)
            const unsigned long long neg1 = f2_pack(-1.f, -1.f);
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
                uint32_t s32[32];
                tmem_ld32(tS + 32 * cc, s32);
                tmem_wait_ld();
                if (nvis < kN) {
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (32 * cc + e >= nvis) s32[e] = __float_as_uint(-INFINITY);
                }
                uint32_t hi[16], lo[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    float x0, x1;
                    f2_unpack(f2_fma(f2_pack(__uint_as_float(s32[2 * e]), __uint_as_float(s32[2 * e + 1])),
                                     c2, nref2),
                              x0, x1);
                    const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
                    const unsigned long long pp = f2_pack(p0, p1);
                    hi[e] = pack_bf16(p0, p1);
                    const unsigned long long hf = f2_pack(__uint_as_float(hi[e] << 16),
                                                          __uint_as_float(hi[e] & 0xffff0000u));
                    float r0, r1;
                    f2_unpack(f2_fma(hf, neg1, pp), r0, r1);
                    lo[e] = pack_bf16(r0, r1);
                }
                tmem_st16(tS + 32 * cc, hi);
                tmem_st16(tS + 32 * cc + 16, lo);
            }
        }
        float sum, sum_hi;
        f2_unpack(sum2, sum, sum_hi);
        sum += sum_hi;
        tmem_wait_st();
        l = l * alpha + sum;
        m_ref = new_ref;
        tc_fence_before_sync();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.p_full[q]);
    }
    if (nk > 0 && ok && wait_all(&sm.pv_done[q], (nk - 1) & 1)) {
        tc_fence_after_sync();
        const float inv = l > 0.f ? 1.f / l : 0.f;
        __nv_bfloat16 *dst = reinterpret_cast<__nv_bfloat16 *>(a.out) +
                             ((size_t)(q0 + tok) * a.Hq + kvh * g + hh) * D;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t o[32];
            tmem_ld32(tO + 32 * cc, o);
            tmem_wait_ld();
            if (valid_row) {
#pragma unroll
                for (int e = 0; e < 32; e += 8) {
                    uint4 w;
                    w.x = pack_bf16(__uint_as_float(o[e]) * inv, __uint_as_float(o[e + 1]) * inv);
                    w.y = pack_bf16(__uint_as_float(o[e + 2]) * inv, __uint_as_float(o[e + 3]) * inv);
                    w.z = pack_bf16(__uint_as_float(o[e + 4]) * inv, __uint_as_float(o[e + 5]) * inv);
                    w.w = pack_bf16(__uint_as_float(o[e + 6]) * inv, __uint_as_float(o[e + 7]) * inv);
                    *reinterpret_cast<uint4 *>(dst + 32 * cc + e) = w;
                }
            }
        }
        if (valid_row && a.lse)
            a.lse[(size_t)(q0 + tok) * a.Hq + kvh * g + hh] =
                l > 0.f ? (m_ref + __log2f(l)) * kLn2P : -INFINITY;
    } else if (nk > 0 && lane == 0) {
        set_error(a.err, GQA_ERR_TIMEOUT);
    }
}

// Longest-first order of the launch's work items.  Item (b, x) is query tiles 2x, 2x+1 of
// sequence b; its cost is the number of 128-key tiles its later query tile reads.  One CTA
// bins the items by cost (a counting sort), then writes them to plan[1..] from the highest
// bin down, and the count to plan[0].  Items of equal cost keep no particular order:
// each is computed on its own, so the outputs do not depend on it.
__global__ void __launch_bounds__(1024)
    prefill_plan_kernel(const PrefillArgs a, const int T, const int items_per_seq) {
    __shared__ __align__(16) int hist[kPlanBins];
    const int total = a.B * items_per_seq;
    // launched with programmatic stream serialization: the inputs and the plan are touched
    // only once the previous kernel in the stream (which may still read the plan) is
    // complete; the prefill CTAs behind this one may become resident from here on
    grid_dependency_wait();
    grid_dependents_launch();
    for (int i = threadIdx.x; i < kPlanBins; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    auto cost_of = [&](int idx, int &item) -> int {
        const int b = idx / items_per_seq, x = idx % items_per_seq;
        const int Lq = a.cu_q[b + 1] - a.cu_q[b];
        if (x * 2 * T >= Lq) return -1;
        const int L = a.seq_lens[b];
        const int last = a.causal ? L - Lq + min(Lq, (x + 1) * 2 * T) - 1 : L - 1;
        item = (b << 16) | x;
        return min(max(last, 0) / kN + 1, kPlanBins - 1);
    };
    for (int idx = threadIdx.x; idx < total; idx += blockDim.x) {
        int item;
        const int c = cost_of(idx, item);
        if (c >= 0) atomicAdd(&hist[c], 1);
        if (idx % items_per_seq == 0) {
            const int b = idx / items_per_seq;
            if (a.cu_q[b + 1] - a.cu_q[b] > a.max_q_len)
                set_error(a.err, GQA_ERR_SHAPE);  // max_q_len below a chunk length
        }
    }
    __syncthreads();
    // exclusive offsets in descending cost order, over the whole block: thread t owns the
    // four bins 4095 - 4t .. 4092 - 4t (one int4, so a warp reads 32 consecutive vectors),
    // then a warp scan and a scan of the warp totals
    static_assert(kPlanBins == 4 * 1024, "four bins per thread of the 1024");
    {
        __shared__ int wsum[32];
        const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
        int4 *h4 = reinterpret_cast<int4 *>(hist);
        const int4 v = h4[kPlanBins / 4 - 1 - t];  // bins (x, y, z, w) = 4092-4t .. 4095-4t
        const int s4 = v.x + v.y + v.z + v.w;
        int incl = s4;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(kAll, incl, o);
            if (lane >= o) incl += u;
        }
        if (lane == 31) wsum[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            const int w = wsum[lane];
            int wi = w;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(kAll, wi, o);
                if (lane >= o) wi += u;
            }
            wsum[lane] = wi - w;  // exclusive offset of each warp
            if (lane == 31) a.plan[0] = wi;
        }
        __syncthreads();
        int run = wsum[warp] + incl - s4;  // bins above this thread's four, in descending order
        int4 o;
        o.w = run;
        run += v.w;
        o.z = run;
        run += v.z;
        o.y = run;
        run += v.y;
        o.x = run;
        h4[kPlanBins / 4 - 1 - t] = o;
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < total; idx += blockDim.x) {
        int item;
        const int c = cost_of(idx, item);
        if (c >= 0) a.plan[1 + atomicAdd(&hist[c], 1)] = item;
    }
}

template <int D>
__global__ void __launch_bounds__(kThreadsP, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                   const __grid_constant__ CUtensorMap qmap, const PrefillArgs a, const int T) {
    extern __shared__ uint8_t smem_raw[];
    constexpr int kHalves = D / 64;
    PSmem<D> &sm = *reinterpret_cast<PSmem<D> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                 ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // block i = (work item i / Hk in the plan's longest-first order, kv head i % Hk), so
    // the longest items are dispatched first, all heads of an item together
    const int kvh = blockIdx.x % a.Hk;
    const int rank = blockIdx.x / a.Hk;
    // launched with programmatic stream serialization behind the plan kernel: nothing is
    // read or written before the plan (and everything before it in the stream) is complete
    grid_dependency_wait();
    if (rank >= a.plan[0]) return;  // uniform for the whole CTA
    const int item = a.plan[1 + rank];
    const int b = item >> 16, ct = item & 0xffff;
    const int g = a.Hq / a.Hk;
    const int q0 = a.cu_q[b];
    const int Lq = a.cu_q[b + 1] - q0;
    const int i0 = ct * kQT * T;  // first token of query tile 0
    if (i0 >= Lq) return;  // uniform for the whole CTA
    const int L = a.seq_lens[b];
    const int P = a.P;
    if (L < Lq || L > a.pt_stride * P) {
        if (threadIdx.x == 0) set_error(a.err, GQA_ERR_BAD_PAGE);
        return;
    }
    // KV tiles each query tile needs (0 when the tile has no token of the chunk)
    int n_kv_q[kQT];
#pragma unroll
    for (int q = 0; q < kQT; ++q) {
        const int ntok = min(T, Lq - (i0 + q * T));
        n_kv_q[q] = ntok <= 0 ? 0
                    : a.causal ? (L - Lq + i0 + q * T + ntok - 1) / kN + 1
                               : (L + kN - 1) / kN;
    }
    const int n_kv = max(n_kv_q[0], n_kv_q[1]);

    if (threadIdx.x == 0) {
        mbar_init(&sm.q_full, 1);
        for (int s = 0; s < kKStages; ++s) {
            mbar_init(&sm.k_full[s], 1);
            mbar_init(&sm.k_empty[s], 1);
        }
        for (int s = 0; s < kVStages; ++s) {
            mbar_init(&sm.v_full[s], 1);
            mbar_init(&sm.v_ready[s], 2);
            mbar_init(&sm.v_empty[s], 1);
        }
        for (int q = 0; q < kQT; ++q) {
            mbar_init(&sm.s_full[q], 1);
            mbar_init(&sm.p_full[q], 4);
            mbar_init(&sm.pv_done[q], 1);
        }
        mbar_init(&sm.mma_done, 1);
        mbar_init(&sm.v_fixsync, 2);
        mbar_init(&sm.v_fix, 1);
        for (int s = 0; s < kVStages; ++s) sm.conv_ovf[s][0] = sm.conv_ovf[s][1] = 0;
        fence_barrier_init();
        fence_proxy_async_smem();
    }
    if (warp == 1) {
        tmem_alloc(&sm.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = sm.tmem_base;

    if (warp >= 4) {
        regs_acquire<kRegsSoftmax>();
        softmax_role<D>(sm, a, tmem, warp, lane, n_kv_q, b, kvh, g, q0, Lq, i0, T, L);
    } else {
    // every warp of warpgroup 0 gives its registers back at the same instruction
    regs_release<kRegsSide>();
    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        const uint64_t pol_kv = policy_evict_last();  // K/V are re-read by the other q tiles
        if (lane == 0) {
            prefetch_tensormap(&qmap);
            prefetch_tensormap(&kmap);
            prefetch_tensormap(&vmap);
            mbar_arrive_expect_tx(&sm.q_full, kQT * kHalves * g * T * 128);
            for (int q = 0; q < kQT; ++q)
                for (int h = 0; h < kHalves; ++h)
                    tma_load_3d(sm.q[q] + h * kHalfBytes, &qmap, &sm.q_full, 64 * h, kvh * g,
                                q0 + i0 + q * T, policy_evict_first());
        }
        const int32_t *pt = a.page_table + (size_t)b * a.pt_stride;
        int issued_k = 0;
        for (int j = 0; j < n_kv; ++j) {
            const int row = kv_chunk_row(a, pt, j, lane, kvh, L);
            const unsigned mask = __ballot_sync(kAll, row >= 0);
            const int ks = j % kKStages, use = j / kKStages;
            bool fail = false;
            if (lane == 0) {
                if (use > 0 && !mbar_wait(&sm.k_empty[ks], (use - 1) & 1)) {
                    set_error(a.err, GQA_ERR_TIMEOUT);
                    fail = true;
                } else {
                    mbar_arrive_expect_tx(&sm.k_full[ks], __popc(mask) * kHalves * kChunkBytes);
                }
            }
            if (__shfl_sync(kAll, fail, 0)) break;
            if (row >= 0) {
#pragma unroll
                for (int h = 0; h < kHalves; ++h)
                    tma_load_2d(sm.k[ks] + h * kHalfBytes + lane * kChunkBytes, &kmap,
                                &sm.k_full[ks], 64 * h, row, pol_kv);
            }
            issued_k = j + 1;
        }
        if (lane == 0) {
            // no copy may outlive the CTA: wait for the Q tiles and the last issued K tiles
            if (!mbar_wait(&sm.q_full, 0)) set_error(a.err, GQA_ERR_TIMEOUT);
            for (int j = max(0, issued_k - kKStages); j < issued_k; ++j)
                if (!mbar_wait(&sm.k_full[j % kKStages], (j / kKStages) & 1)) {
                    set_error(a.err, GQA_ERR_TIMEOUT);
                    break;
                }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        constexpr uint32_t idesc_qk = idesc_bf16_f32(kM, kN, 0, 0);   // Q, K both K-major
        constexpr uint32_t idesc_pv16 = idesc_f16_f32(kM, D, 0, 1);  // P (TMEM), V MN-major
        constexpr uint32_t idesc_pvbf = idesc_bf16_f32(kM, D, 0, 1);
        bool ok = wait_all(&sm.q_full, 0);
        // S_q(j) = Q_q K_j^T into tensor-memory columns [128 q, 128 q + 128)
        auto issue_s = [&](int q, int j) -> bool {
            const int stage = j % kKStages;
            if (!wait_all(&sm.k_full[stage], (j / kKStages) & 1)) return false;
            tc_fence_after_sync();
            if (lane == 0) {
                const uint32_t qa = smem_u32(sm.q[q]), ka = smem_u32(sm.k[stage]);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
                    tc_mma_ss(tmem + 128 * q, smem_desc_sw128(qa + off, 16, 1024),
                              smem_desc_sw128(ka + off, 16, 1024), idesc_qk, kk > 0);
                }
                tc_commit(&sm.s_full[q]);
            }
            __syncwarp();
            return true;
        };
        // O_q += P_q(j) V_j with P_q(j) in S_q's columns: keys 32c..32c+31 as value pairs
        // in columns [32c, 32c+16): f16 against the f16 V tile, or bf16 with the residual
        // pairs in [32c+16, 32c+32) against a V tile that stayed bf16.
        auto issue_pv = [&](int q, int j) -> bool {
            const int stage = j % kVStages;
            if (!wait_all(&sm.p_full[q], j & 1) ||
                !wait_all(&sm.v_ready[stage], (j / kVStages) & 1))
                return false;
            tc_fence_after_sync();
            const bool vbf = sm.v_bf16[stage] != 0;
            if (lane == 0) {
                const uint32_t va = smem_u32(sm.v[stage]);
                const uint32_t tp = tmem + 128 * q, to = tmem + 256 + 128 * q;
                const uint32_t idesc = vbf ? idesc_pvbf : idesc_pv16;
#pragma unroll
                for (int kk = 0; kk < kN / 16; ++kk)
                    tc_mma_ts(to, tp + 32 * (kk >> 1) + 8 * (kk & 1),
                              smem_desc_sw128(va + kk * 2048, kHalfBytes, 1024), idesc,
                              (j > 0 || kk > 0) ? 1u : 0u);
                if (vbf) {
#pragma unroll
                    for (int kk = 0; kk < kN / 16; ++kk)
                        tc_mma_ts(to, tp + 32 * (kk >> 1) + 16 + 8 * (kk & 1),
                                  smem_desc_sw128(va + kk * 2048, kHalfBytes, 1024), idesc_pvbf, 1u);
                }
                tc_commit(&sm.pv_done[q]);
            }
            __syncwarp();
            return true;
        };
        // K tile j is released once the S MMAs that read it are done, V tile j once PV(j)
        for (int q = 0; q < kQT && ok; ++q)
            if (n_kv_q[q] > 0) ok = issue_s(q, 0);
        if (ok && lane == 0 && n_kv > 0) tc_commit(&sm.k_empty[0]);
        __syncwarp();
        for (int j = 0; j < n_kv && ok; ++j) {
            for (int q = 0; q < kQT && ok; ++q) {
                if (j >= n_kv_q[q]) continue;
                ok = issue_pv(q, j);
                if (ok && j + 1 < n_kv_q[q]) ok = issue_s(q, j + 1);
            }
            if (ok && lane == 0) {
                tc_commit(&sm.v_empty[j % kVStages]);
                if (j + 1 < n_kv) tc_commit(&sm.k_empty[(j + 1) % kKStages]);
            }
            __syncwarp();
        }
        if (!ok && lane == 0) set_error(a.err, GQA_ERR_TIMEOUT);
        // every MMA issued must be finished before tensor memory is released
        if (lane == 0) tc_commit(&sm.mma_done);
        __syncwarp();
        if (!wait_all(&sm.mma_done, 0) && lane == 0) set_error(a.err, GQA_ERR_TIMEOUT);
    } else {
        // ------------------------------------------------------------ V loads + converters
        // Warp 2 also copies the V tiles in (one lane per 16-key chunk): the first
        // kVStages at once, then, after converting tile j, it waits for PV(j - 1) to free
        // that tile's stage and loads tile j + kVStages - 1 into it.
        const int cid = threadIdx.x - 64;  // 0..63
        const int cw = warp - 2;
        constexpr int kChunks16 = tile_bytes<D>() / 16;  // 16-byte chunks of a V tile
        const int32_t *pt = a.page_table + (size_t)b * a.pt_stride;
        const uint64_t pol_kv = policy_evict_last();
        int issued_v = 0;
        // V tile jv into its stage, counted on `bar`
        auto load_v_to = [&](int jv, uint64_t *bar) {
            const int row = kv_chunk_row(a, pt, jv, lane, kvh, L);
            const unsigned mask = __ballot_sync(kAll, row >= 0);
            const int vs = jv % kVStages;
            if (lane == 0) mbar_arrive_expect_tx(bar, __popc(mask) * kHalves * kChunkBytes);
            __syncwarp();
            if (row >= 0) {
#pragma unroll
                for (int h = 0; h < kHalves; ++h)
                    tma_load_2d(sm.v[vs] + h * kHalfBytes + lane * kChunkBytes, &vmap, bar, 64 * h, row,
                                pol_kv);
            }
        };
        auto load_v = [&](int jv) {
            load_v_to(jv, &sm.v_full[jv % kVStages]);
            issued_v = jv + 1;
        };
        int nfix = 0;  // V tiles copied again so far (the same count in both converter warps)
        if (cw == 0)
            for (int jv = 0; jv < min(n_kv, kVStages); ++jv) load_v(jv);
        for (int j = 0; j < n_kv; ++j) {
            const int stage = j % kVStages;
            if (!wait_all(&sm.v_full[stage], (j / kVStages) & 1)) {
                if (lane == 0) set_error(a.err, GQA_ERR_TIMEOUT);
                break;
            }
            uint8_t *vt = sm.v[stage];
            // Each thread owns chunks cid, cid + 64, ... (chunk c: half c / 1024, key row
            // (c / 8) % 128).  On the sequence's last tile the keys at or past L (which hold
            // anything, even NaN) become zero first, so their zero weights add exactly zero
            // (zero has the same bits in bf16 and f16).  Then every chunk becomes f16 in place
            // (bf16 -> fp32 is exact; fp32 -> f16 rounds to nearest, magnitudes under 2^-14
            // becoming f16 subnormals).  A value beyond the f16 range (or Inf / NaN) comes out
            // with all exponent bits set: the largest magnitude of the results shows it.
            const int valid = L - j * kN;
            if (valid < kN) {
                for (int c = cid; c < kChunks16; c += kConvThreads)
                    if (((c >> 3) & (kN - 1)) >= valid)
                        *reinterpret_cast<uint4 *>(vt + 16 * c) = make_uint4(0u, 0u, 0u, 0u);
            }
            uint32_t mx = 0u;
            constexpr int kBatch = 8;  // chunks in flight per thread
#pragma unroll 1
            for (int c0 = cid; c0 < kChunks16; c0 += kBatch * kConvThreads) {
                uint4 w[kBatch];
#pragma unroll
                for (int i = 0; i < kBatch; ++i)
                    w[i] = *reinterpret_cast<const uint4 *>(vt + 16 * (c0 + i * kConvThreads));
#pragma unroll
                for (int i = 0; i < kBatch; ++i) {
                    w[i].x = pack_f16(__uint_as_float(w[i].x << 16), __uint_as_float(w[i].x & 0xffff0000u));
                    w[i].y = pack_f16(__uint_as_float(w[i].y << 16), __uint_as_float(w[i].y & 0xffff0000u));
                    w[i].z = pack_f16(__uint_as_float(w[i].z << 16), __uint_as_float(w[i].z & 0xffff0000u));
                    w[i].w = pack_f16(__uint_as_float(w[i].w << 16), __uint_as_float(w[i].w & 0xffff0000u));
                    mx = umax16x2(mx, umax16x2(umax16x2(w[i].x & 0x7fff7fffu, w[i].y & 0x7fff7fffu),
                                               umax16x2(w[i].z & 0x7fff7fffu, w[i].w & 0x7fff7fffu)));
                    *reinterpret_cast<uint4 *>(vt + 16 * (c0 + i * kConvThreads)) = w[i];
                }
            }
            const bool big = (mx & 0xffffu) >= 0x7c00u || (mx >> 16) >= 0x7c00u;
            // exchange the range decision with the other converter warp: (j + 1) * 2 + flag, and a
            // bounded wait for the partner's entry of this tile
            const int mine = ((j + 1) << 1) | (__any_sync(kAll, big) ? 1 : 0);
            volatile int *xo = &sm.conv_ovf[stage][0];
            if (lane == 0) xo[cw] = mine;
            int theirs = xo[cw ^ 1];
            if ((theirs >> 1) != j + 1) {
                const unsigned long long t0 = global_timer_ns();
                while ((theirs >> 1) != j + 1 && global_timer_ns() - t0 < kWaitLimitNs) theirs = xo[cw ^ 1];
            }
            if (__any_sync(kAll, (theirs >> 1) != j + 1)) {
                if (lane == 0) set_error(a.err, GQA_ERR_TIMEOUT);
                break;
            }
            const bool keep_bf16 = ((mine | theirs) & 1) != 0;
            if (keep_bf16) {
                // Copy tile j again (bf16) once both warps' f16 stores are ordered before the
                // copy: each warp fences them for the async proxy and arrives on v_fixsync, and
                // warp 2 issues the copy after both arrivals.  Then the keys past L become zero
                // again.
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.v_fixsync);
                bool fixed = true;
                if (cw == 0) {
                    fixed = wait_all(&sm.v_fixsync, nfix & 1);
                    if (fixed) load_v_to(j, &sm.v_fix);
                }
                if (!fixed || !wait_all(&sm.v_fix, nfix & 1)) {
                    if (lane == 0) set_error(a.err, GQA_ERR_TIMEOUT);
                    break;
                }
                ++nfix;
                if (valid < kN)
                    for (int c = cid; c < kChunks16; c += kConvThreads)
                        if (((c >> 3) & (kN - 1)) >= valid)
                            *reinterpret_cast<uint4 *>(vt + 16 * c) = make_uint4(0u, 0u, 0u, 0u);
            }
            // the tensor core (async proxy) reads what these generic stores wrote
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                if (cw == 0) sm.v_bf16[stage] = keep_bf16 ? 1 : 0;
                mbar_arrive(&sm.v_ready[stage]);
            }
            // stage of tile j - 1 -> tile j + kVStages - 1, once PV(j - 1) has read it
            if (cw == 0 && j >= 1 && j + kVStages - 1 < n_kv) {
                if (!wait_all(&sm.v_empty[(j - 1) % kVStages], ((j - 1) / kVStages) & 1)) {
                    if (lane == 0) set_error(a.err, GQA_ERR_TIMEOUT);
                    break;
                }
                load_v(j + kVStages - 1);
            }
        }
        // no copy may outlive the CTA
        if (cw == 0 && lane == 0)
            for (int j = max(0, issued_v - kVStages); j < issued_v; ++j)
                if (!mbar_wait(&sm.v_full[j % kVStages], (j / kVStages) & 1)) {
                    set_error(a.err, GQA_ERR_TIMEOUT);
                    break;
                }
    }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, 512);
    }
}

template <int D>
cudaError_t launch_prefill_d(const PrefillArgs &a, const CUtensorMap &kmap, const CUtensorMap &vmap,
                             const CUtensorMap &qmap, cudaStream_t stream) {
    const int g = a.Hq / a.Hk;
    const int T = kM / g;
    const size_t smem = sizeof(PSmem<D>) + 1024;
    cudaError_t e = cudaFuncSetAttribute(prefill_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const int items_per_seq = (a.max_q_len + kQT * T - 1) / (kQT * T);
    if (items_per_seq == 0 || a.B == 0) return cudaSuccess;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t pc = {};
    pc.gridDim = dim3(1);
    pc.blockDim = dim3(1024);
    pc.stream = stream;
    pc.attrs = attr;
    pc.numAttrs = 1;
    if ((e = cudaLaunchKernelEx(&pc, prefill_plan_kernel, a, T, items_per_seq)) != cudaSuccess) return e;
    cudaLaunchConfig_t kc = pc;
    kc.gridDim = dim3(a.B * items_per_seq * a.Hk);
    kc.blockDim = dim3(kThreadsP);
    kc.dynamicSmemBytes = smem;
    return cudaLaunchKernelEx(&kc, prefill_kernel<D>, kmap, vmap, qmap, a, T);
}

}  // namespace

cudaError_t launch_prefill(const PrefillArgs &a, const CUtensorMap &kmap, const CUtensorMap &vmap,
                           const CUtensorMap &qmap, cudaStream_t stream) {
    return a.D == 64 ? launch_prefill_d<64>(a, kmap, vmap, qmap, stream)
                     : launch_prefill_d<128>(a, kmap, vmap, qmap, stream);
}

}  // namespace gqa
