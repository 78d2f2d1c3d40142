// Lightning-indexer scores for decode-style calls (one query per sequence).
//
// Computes the same score as the fused prefill kernel (indexer.cuh):
//     I[b,s] = k_scale[s] * sum_j (w[b,j] * q_scale[b]) * ReLU(q_I[b,j,:] . k_I[s,:])
// for every visible key s of every sequence b, and writes the order-preserving
// key of I[b,s] to a per-sequence score row in the workspace. With one query
// per sequence the streaming top-k has nothing to stream over across queries:
// each chunk of keys that is no longer than k keeps all of its keys as
// candidates, so the candidate list of a chunk is its dense score vector, and
// topk_rows_kernel then selects the k winners of each row once. What is stored
// is one score per (sequence, key), never a query x key matrix.
//
// Mapping to Blackwell:
//  * Work item = (sequence, chunk of IDX_DEC_CHUNK key tiles), dealt to
//    persistent CTAs in a snake. The sequence's q_I block (64 heads, operand
//    B) is loaded by TMA into one of two slots; key tiles (operand A, 128
//    keys) stream through a TMA ring (128-byte swizzle, no multicast).
//  * One MMA per tile, M = 128 keys x N = 64 heads x K = d_I, into an 8-deep
//    ring of 64-column TMEM accumulators.
//  * Four epilogue warpgroups take the tiles round robin (tile i -> warpgroup
//    i % 4), each reading its accumulator with the 16x256b TMEM shape: a
//    thread holds 16 heads of 4 keys and its 16 head weights in registers,
//    and a 3-shuffle reduce-scatter over the 4 lanes sharing the keys
//    finishes the head sum.
//
// Warp roles: warp 0 TMA producer, warp 1 MMA issuer, warp 2 TMEM allocator,
// warp 3 idle, warps 4-19 the epilogue warpgroups.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"
#include "topk_select.cuh"

namespace ic {

constexpr int IDX_DEC_CHUNK = 8;   // key tiles (of 128) per work item
constexpr int IDX_DEC_ACC = 8;     // TMEM accumulator stages of 64 columns

struct IdxDecParams {
    const void* w;            // [batch, H_I] bf16 or fp32
    const float* q_scale;     // [batch] or null
    const float* k_scale;     // [batch, n_k] or null
    int w_is_f32;
    int batch, n_k, n_vis;    // n_vis = keys visible to every query
    int n_chunks;             // chunks per sequence
    int n_work;               // batch * n_chunks
    int stride;               // score-row stride (keys)
    uint32_t* scores;         // [batch, stride] order-preserving score keys
};

template <int DI_, bool FP8_, int STAGES_>
struct IdxDecCfg {
    static constexpr int HI = 64, DI = DI_, STAGES = STAGES_;
    static constexpr bool FP8 = FP8_;
    static constexpr int ESZ = FP8 ? 1 : 2;
    static constexpr int ROW_BYTES = DI * ESZ;
    static_assert(ROW_BYTES % 128 == 0, "rows must be whole 128-byte swizzle atoms");
    static constexpr int KATOMS = ROW_BYTES / 128;
    static constexpr int ATOM_ELEMS = 128 / ESZ;
    static constexpr int KSTEPS = ROW_BYTES / 32;
    static constexpr int THREADS = 128 + 4 * 128;
    // setmaxnreg split of the launch's 96 registers per thread (65536 / 640,
    // in steps of 8): the TMA/MMA warpgroup drops to 32, the epilogue takes 112
    static constexpr int REGS_LAUNCH = 96, REGS_CTRL = 32, REGS_EPI = 112;
    static_assert(128 * REGS_CTRL + 512 * REGS_EPI <= REGS_LAUNCH * THREADS, "register split");
    static constexpr int Q_BYTES = HI * ROW_BYTES;
    static constexpr int K_BYTES = 128 * ROW_BYTES;
    static constexpr uint32_t IDESC = make_idesc(128, HI, FP8 ? FMT_E4M3 : FMT_BF16, FP8 ? FMT_E4M3 : FMT_BF16);
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + 2 * Q_BYTES;
    static constexpr int OFF_BAR = OFF_K + STAGES * K_BYTES;
    // mbarrier slots: k_full[STAGES], k_empty[STAGES], q_full[2], q_empty[2],
    // acc_full[ACC], acc_empty[ACC], drain (the abort teardown's MMA drain)
    static constexpr int NUM_BARS = 2 * STAGES + 4 + 2 * IDX_DEC_ACC + 1;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int SMEM_BYTES = OFF_MISC + 16;
    static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;
    static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
};

struct IdxDecWork {
    int b, t0, n_tiles;
};

__device__ __forceinline__ IdxDecWork idx_dec_work(const IdxDecParams& p, int item) {
    IdxDecWork w;
    w.b = item / p.n_chunks;
    const int c = item % p.n_chunks;
    w.t0 = c * IDX_DEC_CHUNK;
    const int tiles = ceil_div(p.n_vis, 128);
    w.n_tiles = max(0, min(IDX_DEC_CHUNK, tiles - w.t0));
    return w;
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
    indexer_decode_scores_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                                 const IdxDecParams p) {
    constexpr int HI = Cfg::HI;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align_smem_1024(smem_raw);
    const uint32_t s_base = smem_u32(smem);
    const uint32_t bar0 = s_base + Cfg::OFF_BAR;
    auto bar_k_full = [&](int s) { return bar0 + 8u * s; };
    auto bar_k_empty = [&](int s) { return bar0 + 8u * (Cfg::STAGES + s); };
    auto bar_q_full = [&](int s) { return bar0 + 8u * (2 * Cfg::STAGES + s); };
    auto bar_q_empty = [&](int s) { return bar0 + 8u * (2 * Cfg::STAGES + 2 + s); };
    auto bar_acc_full = [&](int a) { return bar0 + 8u * (2 * Cfg::STAGES + 4 + a); };
    auto bar_acc_empty = [&](int a) { return bar0 + 8u * (2 * Cfg::STAGES + 4 + IDX_DEC_ACC + a); };
    const uint32_t bar_drain = bar0 + 8u * (2 * Cfg::STAGES + 4 + 2 * IDX_DEC_ACC);
    static_assert(Cfg::NUM_BARS == 2 * Cfg::STAGES + 4 + 2 * IDX_DEC_ACC + 1, "barrier slots");
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::OFF_MISC + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < Cfg::STAGES; ++s) {
            mbar_init(bar_k_full(s), 1);
            mbar_init(bar_k_empty(s), 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar_q_full(s), 1);
            mbar_init(bar_q_empty(s), 1);
        }
        for (int a = 0; a < IDX_DEC_ACC; ++a) {
            mbar_init(bar_acc_full(a), 1);
            mbar_init(bar_acc_empty(a), 4);  // the four warps of the owning warpgroup
        }
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
    }
    if (warp == 2) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const int n_rounds = ceil_div(p.n_work, static_cast<int>(gridDim.x));
    // copies issued by the producer: Q loads armed, K tiles armed (counts)
    uint32_t q_armed = 0, k_armed = 0;
    auto snake = [&](int r) {
        return r * static_cast<int>(gridDim.x) + ((r & 1) ? (static_cast<int>(gridDim.x) - 1 - static_cast<int>(blockIdx.x))
                                                          : static_cast<int>(blockIdx.x));
    };

    if (warp < 4) {
        regs_dec<Cfg::REGS_CTRL>();
        if (warp == 0 && lane == 0) {
            // ------------------------------------------------------------ producer
            uint32_t kst = 0, qit = 0;
            for (int r = 0; r < n_rounds; ++r) {
                const int item = snake(r);
                if (item >= p.n_work) continue;
                const IdxDecWork wk = idx_dec_work(p, item);
                if (wk.n_tiles == 0) continue;
                const int qs = qit & 1;
                // a wait that fails means the CTA aborted: nothing more is issued
                if (mbar_wait(bar_q_empty(qs), ((qit >> 1) & 1) ^ 1, abort_flag)) {
                    mbar_arrive_expect_tx(bar_q_full(qs), Cfg::Q_BYTES);
#pragma unroll
                    for (int a = 0; a < Cfg::KATOMS; ++a)
                        tma_load_2d(s_base + Cfg::OFF_Q + qs * Cfg::Q_BYTES + a * HI * 128, &tm_q,
                                    bar_q_full(qs), a * Cfg::ATOM_ELEMS, wk.b * HI);
                    q_armed = qit + 1;
                }
                ++qit;
                for (int t = 0; t < wk.n_tiles; ++t) {
                    const int s = kst % Cfg::STAGES;
                    if (mbar_wait(bar_k_empty(s), ((kst / Cfg::STAGES) & 1) ^ 1, abort_flag)) {
                        mbar_arrive_expect_tx(bar_k_full(s), Cfg::K_BYTES);
                        const int krow = wk.b * p.n_k + (wk.t0 + t) * 128;
#pragma unroll
                        for (int a = 0; a < Cfg::KATOMS; ++a)
                            tma_load_2d(s_base + Cfg::OFF_K + s * Cfg::K_BYTES + a * 128 * 128, &tm_k,
                                        bar_k_full(s), a * Cfg::ATOM_ELEMS, krow);
                        k_armed = kst + 1;
                    }
                    ++kst;
                }
            }
        } else if (warp == 1 && lane == 0) {
            // ------------------------------------------------------------ MMA issuer
            uint32_t kst = 0, qit = 0, seq = 0;
            for (int r = 0; r < n_rounds; ++r) {
                const int item = snake(r);
                if (item >= p.n_work) continue;
                const IdxDecWork wk = idx_dec_work(p, item);
                if (wk.n_tiles == 0) continue;
                const int qs = qit & 1;
                mbar_wait(bar_q_full(qs), (qit >> 1) & 1, abort_flag);
                tc_fence_after();
                const uint64_t bdesc0 = make_sw128_desc(s_base + Cfg::OFF_Q + qs * Cfg::Q_BYTES);
                for (int t = 0; t < wk.n_tiles; ++t) {
                    const int s = kst % Cfg::STAGES;
                    const int a = seq % IDX_DEC_ACC;
                    const bool go = mbar_wait(bar_k_full(s), (kst / Cfg::STAGES) & 1, abort_flag) &&
                                    mbar_wait(bar_acc_empty(a), ((seq / IDX_DEC_ACC) & 1) ^ 1, abort_flag);
                    tc_fence_after();
                    if (!go) {  // aborted: issue nothing more; the teardown drains
                        ++kst;
                        ++seq;
                        continue;
                    }
                    const uint64_t adesc0 = make_sw128_desc(s_base + Cfg::OFF_K + s * Cfg::K_BYTES);
#pragma unroll
                    for (int ks = 0; ks < Cfg::KSTEPS; ++ks) {
                        const int atom = ks >> 2;
                        const uint32_t koff = (ks & 3) * 32;
                        const uint64_t adesc = adesc0 + ((atom * 128 * 128 + koff) >> 4);
                        const uint64_t bdesc = bdesc0 + ((atom * HI * 128 + koff) >> 4);
                        if constexpr (Cfg::FP8)
                            mma_f8(tmem_base + a * HI, adesc, bdesc, Cfg::IDESC, ks > 0 ? 1u : 0u);
                        else
                            mma_f16(tmem_base + a * HI, adesc, bdesc, Cfg::IDESC, ks > 0 ? 1u : 0u);
                    }
                    mma_commit(bar_k_empty(s));
                    mma_commit(bar_acc_full(a));
                    ++kst;
                    ++seq;
                }
                mma_commit(bar_q_empty(qs));
                ++qit;
            }
        }
    } else {
        regs_inc<Cfg::REGS_EPI>();
        // ------------------------------------------------------------ epilogue
        // the score rows go to the caller's workspace, which the previous
        // kernel of a layer loop may still be using
        griddep_sync();
        const int e = (warp - 4) >> 2;  // warpgroup: tiles with seq % 4 == e
        const int wq = warp & 3;        // TMEM lane quarter
        const int c4 = lane & 3, r8 = lane >> 2;
        // key (within the warp's 32) held after the reduce-scatter
        const int kidx = r8 + 8 * (2 * (c4 & 1) + (c4 >> 1));
        uint32_t seq = 0;
        for (int r = 0; r < n_rounds; ++r) {
            const int item = snake(r);
            if (item >= p.n_work) continue;
            const IdxDecWork wk = idx_dec_work(p, item);
            if (wk.n_tiles == 0) continue;
            // this lane's 16 head weights of the sequence, with its query scale
            float2 wreg[8];
            const float qsc = p.q_scale ? p.q_scale[wk.b] : 1.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int64_t h = static_cast<int64_t>(wk.b) * HI + 8 * i + 2 * c4;
                float w0, w1;
                if (p.w_is_f32) {
                    w0 = static_cast<const float*>(p.w)[h];
                    w1 = static_cast<const float*>(p.w)[h + 1];
                } else {
                    w0 = __bfloat162float(static_cast<const __nv_bfloat16*>(p.w)[h]);
                    w1 = __bfloat162float(static_cast<const __nv_bfloat16*>(p.w)[h + 1]);
                }
                wreg[i] = make_float2(w0 * qsc, w1 * qsc);
            }
            uint32_t* srow = p.scores + static_cast<int64_t>(wk.b) * p.stride;
            for (int t = 0; t < wk.n_tiles; ++t, ++seq) {
                if (static_cast<int>(seq & 3) != e) continue;
                const int a = seq % IDX_DEC_ACC;
                const int s_key = (wk.t0 + t) * 128 + wq * 32 + kidx;
                const bool in_range = s_key < p.n_vis;
                const float ksc = (p.k_scale != nullptr && in_range)
                                      ? p.k_scale[static_cast<int64_t>(wk.b) * p.n_k + s_key]
                                      : 1.f;
                mbar_wait(bar_acc_full(a), (seq / IDX_DEC_ACC) & 1, abort_flag);
                tc_fence_after();
                uint32_t ra[32], rb[32];
                const uint32_t tb = tmem_base + (static_cast<uint32_t>(wq * 32) << 16) + a * HI;
                tmem_ld_16x256b_x8(tb, ra);
                tmem_ld_16x256b_x8(tb + (16u << 16), rb);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_acc_empty(a));
                float2 acc[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) acc[u] = make_float2(0.f, 0.f);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    auto relu2 = [](uint32_t x, uint32_t y) {
                        return make_float2(fmaxf(__uint_as_float(x), 0.f), fmaxf(__uint_as_float(y), 0.f));
                    };
                    acc[0] = __ffma2_rn(wreg[i], relu2(ra[4 * i], ra[4 * i + 1]), acc[0]);      // key r
                    acc[1] = __ffma2_rn(wreg[i], relu2(ra[4 * i + 2], ra[4 * i + 3]), acc[1]);  // key r + 8
                    acc[2] = __ffma2_rn(wreg[i], relu2(rb[4 * i], rb[4 * i + 1]), acc[2]);      // key r + 16
                    acc[3] = __ffma2_rn(wreg[i], relu2(rb[4 * i + 2], rb[4 * i + 3]), acc[3]);  // key r + 24
                }
                const float p0 = acc[0].x + acc[0].y, p1 = acc[1].x + acc[1].y;
                const float p2 = acc[2].x + acc[2].y, p3 = acc[3].x + acc[3].y;
                const bool odd = (c4 & 1) != 0;
                const float q0 = (odd ? p2 : p0) + __shfl_xor_sync(0xffffffffu, odd ? p0 : p2, 1);
                const float q1 = (odd ? p3 : p1) + __shfl_xor_sync(0xffffffffu, odd ? p1 : p3, 1);
                const bool hi2 = (c4 & 2) != 0;
                const float sum = (hi2 ? q1 : q0) + __shfl_xor_sync(0xffffffffu, hi2 ? q0 : q1, 2);
                if (in_range) srow[s_key] = float_to_ordered(sum * ksc);
            }
        }
    }

    // ---------------------------------------------------------------- teardown
    __syncthreads();
    if (*abort_flag) {  // final after the barrier: the same in every thread
        if (warp == 0 && lane == 0) {
            for (uint32_t i = q_armed > 2 ? q_armed - 2 : 0; i < q_armed; ++i)
                mbar_drain(bar_q_full(i & 1), (i >> 1) & 1);
            for (uint32_t i = k_armed > Cfg::STAGES ? k_armed - Cfg::STAGES : 0; i < k_armed; ++i)
                mbar_drain(bar_k_full(i % Cfg::STAGES), (i / Cfg::STAGES) & 1);
        }
        if (warp == 1 && lane == 0) {
            mma_commit(bar_drain);
            mbar_drain(bar_drain, 0);
        }
        __syncthreads();
    }
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

// Exact top-k of each score row written by indexer_decode_scores_kernel, by
// radix select on the order-preserving score keys. A row belongs to one
// cluster of TOPK_ROWS_CL CTAs: CTA c holds keys [8192 c, 8192 c + 8192),
// thread t of it keys [8192 c + 8 t, 8192 c + 8 t + 8), in registers.
//  * The cluster's min / max gives the row's key range [kmin, kmax]; the
//    select works on d = key - kmin, whose bit length is at most 32.
//  * Each pass takes the next 12 (or fewer) bits of d below those already
//    fixed. Every CTA histograms its keys that match the fixed high bits in
//    its own shared memory; each then sums the cluster's histograms through
//    distributed shared memory and, with a block scan from the top, finds the
//    bin that holds the k-th largest key and how many keys of that bin are
//    still to be taken. Every CTA computes the same sums, so all take the same
//    path. At most three passes fix every bit, giving the k-th largest key T.
//  * A packed scan of (keys > T, keys == T) per thread, offset by the counts
//    of the lower-ranked CTAs, then writes the winners: every key above T and
//    the lowest-indexed keys equal to T, in ascending key order. Ties thus go
//    to the lower key; -1 pads rows with fewer than k visible keys.
constexpr int TOPK_ROWS_NT = 1024;
constexpr int TOPK_ROWS_CL = 4;  // CTAs per row (one cluster)
constexpr int TOPK_ROWS_E = 8;   // keys per thread
constexpr int TOPK_ROWS_CTA = TOPK_ROWS_NT * TOPK_ROWS_E;
constexpr int TOPK_ROWS_MAX = TOPK_ROWS_CL * TOPK_ROWS_CTA;
constexpr int TOPK_RADIX_BITS = 12;
constexpr int TOPK_RADIX_BINS = 1 << TOPK_RADIX_BITS;
static_assert(TOPK_RADIX_BINS == 4 * TOPK_ROWS_NT, "four histogram bins per thread");
static_assert(TOPK_ROWS_MAX == 32768, "rows of up to 32768 keys");

// Inclusive sum over the 1024 threads of the block, in thread order; `total`
// gets the block's sum. `red` is 32 words of shared memory, free again when
// the call returns.
__device__ __forceinline__ uint32_t block_scan_1024(uint32_t v, uint32_t* red, uint32_t& total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    if (lane == 31) red[warp] = v;
    __syncthreads();
    if (warp == 0) {
        uint32_t w = red[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t n = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += n;
        }
        red[lane] = w;
    }
    __syncthreads();
    total = red[31];
    const uint32_t before = warp > 0 ? red[warp - 1] : 0u;
    __syncthreads();
    return v + before;
}

__global__ void __cluster_dims__(TOPK_ROWS_CL, 1, 1) __launch_bounds__(TOPK_ROWS_NT)
    topk_rows_kernel(const uint32_t* __restrict__ scores, int stride, int n_vis, int topk,
                     int32_t* __restrict__ idx_out) {
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    // two histograms, alternating between passes: a CTA rewrites one only
    // after every CTA of the cluster has passed the next pass's barrier, so
    // after the last remote read of it
    __shared__ __align__(16) uint32_t hist2[2][TOPK_RADIX_BINS];
    __shared__ uint32_t red[32];
    __shared__ uint32_t mm[2][32];
    __shared__ uint32_t pick[2];  // bin holding the k-th key, keys of it still to take
    // read by the other CTAs of the cluster: this CTA's key min and max, and
    // its packed count of (keys == T) << 16 | (keys > T)
    __shared__ uint32_t xch[3];
    const int crank = static_cast<int>(cluster.block_rank());
    const int row = blockIdx.x / TOPK_ROWS_CL;
    const int tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    griddep_sync();  // the score rows come from the previous kernel
    int32_t* out = idx_out + static_cast<int64_t>(row) * topk;
    if (n_vis <= topk) {  // every visible key wins (uniform across the cluster)
        for (int i = crank * TOPK_ROWS_NT + tid; i < topk; i += TOPK_ROWS_CL * TOPK_ROWS_NT)
            out[i] = i < n_vis ? i : -1;
        return;
    }
    // this thread's keys; stride is a multiple of 128 keys and at least n_vis,
    // so an 8-key chunk that starts inside the row ends inside it too
    const int i0 = crank * TOPK_ROWS_CTA + tid * TOPK_ROWS_E;
    const int nv = min(max(n_vis - i0, 0), TOPK_ROWS_E);  // its first nv keys are visible
    uint32_t key[TOPK_ROWS_E];
    if (nv > 0) {
        const uint4* src = reinterpret_cast<const uint4*>(scores + static_cast<int64_t>(row) * stride + i0);
#pragma unroll
        for (int j = 0; j < TOPK_ROWS_E / 4; ++j) {
            const uint4 v = __ldg(src + j);
            key[4 * j] = v.x;
            key[4 * j + 1] = v.y;
            key[4 * j + 2] = v.z;
            key[4 * j + 3] = v.w;
        }
    } else {
#pragma unroll
        for (int j = 0; j < TOPK_ROWS_E; ++j) key[j] = 0u;
    }
    // key range of the row: this CTA's, then the cluster's
    uint32_t kmin = 0xffffffffu, kmax = 0u;
#pragma unroll
    for (int j = 0; j < TOPK_ROWS_E; ++j) {
        if (j < nv) {
            kmin = min(kmin, key[j]);
            kmax = max(kmax, key[j]);
        }
    }
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    if (lane == 0) {
        mm[0][warp] = kmin;
        mm[1][warp] = kmax;
    }
    __syncthreads();
    if (warp == 0) {
        kmin = __reduce_min_sync(0xffffffffu, mm[0][lane]);
        kmax = __reduce_max_sync(0xffffffffu, mm[1][lane]);
        if (lane == 0) {
            xch[0] = kmin;
            xch[1] = kmax;
        }
    }
    cluster.sync();
    kmin = 0xffffffffu;
    kmax = 0u;
#pragma unroll
    for (int c = 0; c < TOPK_ROWS_CL; ++c) {
        const uint32_t* x = cluster.map_shared_rank(xch, c);
        kmin = min(kmin, x[0]);
        kmax = max(kmax, x[1]);
    }

    // radix passes over d = key - kmin, high bits first
    int hi = 32 - __clz(kmax - kmin);  // bits of d not fixed yet (0: every key equal)
    uint32_t prefix = 0u;               // the fixed bits of the k-th largest d
    uint32_t k_rem = static_cast<uint32_t>(topk);
    int npass = 0;
    while (hi > 0) {  // uniform across the cluster
        uint32_t* hist = hist2[npass++ & 1];
        const int lo = max(0, hi - TOPK_RADIX_BITS);
        const uint32_t mask = (1u << (hi - lo)) - 1u;
#pragma unroll
        for (int q = 0; q < 4; ++q) hist[4 * tid + q] = 0u;
        __syncthreads();
#pragma unroll
        for (int j = 0; j < TOPK_ROWS_E; ++j) {
            const uint32_t d = key[j] - kmin;
            if (j < nv && (static_cast<uint64_t>(d) >> hi) == prefix) atomicAdd(&hist[(d >> lo) & mask], 1u);
        }
        cluster.sync();  // every CTA's histogram is complete
        uint32_t h4[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int c = 0; c < TOPK_ROWS_CL; ++c) {
            const uint4 v = *reinterpret_cast<const uint4*>(cluster.map_shared_rank(hist, c) + 4 * tid);
            h4[0] += v.x;
            h4[1] += v.y;
            h4[2] += v.z;
            h4[3] += v.w;
        }
        uint32_t total;
        const uint32_t incl = block_scan_1024(h4[0] + h4[1] + h4[2] + h4[3], red, total);
        uint32_t above = total - incl;  // keys in the bins of higher threads
#pragma unroll
        for (int q = 3; q >= 0; --q) {
            if (above < k_rem && k_rem <= above + h4[q]) {
                pick[0] = static_cast<uint32_t>(4 * tid + q);
                pick[1] = k_rem - above;
            }
            above += h4[q];
        }
        __syncthreads();
        prefix = (prefix << (hi - lo)) | pick[0];
        k_rem = pick[1];
        hi = lo;
        __syncthreads();  // pick is rewritten by the next pass
    }
    const uint32_t T = kmin + prefix;  // the k-th largest key; k_rem keys equal to it win

    // winners in key order: a packed scan of (keys above T, keys equal to T),
    // offset by the packed counts of the lower-ranked CTAs
    uint32_t gt = 0, eq = 0;
#pragma unroll
    for (int j = 0; j < TOPK_ROWS_E; ++j) {
        if (j < nv) {
            gt += key[j] > T ? 1u : 0u;
            eq += key[j] == T ? 1u : 0u;
        }
    }
    uint32_t total;
    const uint32_t packed = (eq << 16) | gt;  // each half sums to at most 32768 over the row
    uint32_t excl = block_scan_1024(packed, red, total) - packed;
    if (tid == 0) xch[2] = total;
    cluster.sync();
    for (int c = 0; c < crank; ++c) excl += cluster.map_shared_rank(xch, c)[2];
    uint32_t tie = excl >> 16;
    int pos = static_cast<int>((excl & 0xffffu) + min(tie, k_rem));
#pragma unroll
    for (int j = 0; j < TOPK_ROWS_E; ++j) {
        if (j < nv) {
            bool take = key[j] > T;
            if (key[j] == T) {
                take = tie < k_rem;
                ++tie;
            }
            if (take) {
                if (IC_DCHECK(pos < topk)) out[pos] = i0 + j;
                ++pos;
            }
        }
    }
    cluster.sync();  // no CTA leaves while another may still read its xch
}

}  // namespace ic
