// Fused lightning indexer + streaming top-k for sm_100a.
//
// What it computes (IndexCache paper, Abstract: "a lightweight lightning
// indexer selects the top-k most relevant tokens per query"; score of the DSA
// lightning indexer):
//     I[t,s] = k_scale[s] * sum_j (w[t,j] * q_scale[t]) * ReLU(X[t,j,s]),
//     X[t,j,s] = q_I[t,j,:] . k_I[s,:]  (raw bf16 / E4M3 operands),
// and for every query the top-k keys s <= t by (I desc, s asc).
// Positive per-token scales factor out of the ReLU, so the product of the
// scales and the raw-operand dot product equals the dot product of the
// dequantised operands.
//
// Mapping to Blackwell:
//  * The contraction X is a dense GEMM on the tcgen05 tensor cores: M = 128
//    keys (TMEM lanes), N = G queries x H_I heads, K = d_I. The key tile
//    (operand A) streams through a TMA ring (128B swizzle, no multicast); the
//    G queries' q_I rows (operand B) stay resident for the whole key sweep.
//    Accumulators live in TMEM, double-buffered, so the MMA of tile i+1 runs
//    while the epilogue reads tile i.
//  * Epilogue: each thread owns one key (one TMEM lane) and reduces its
//    heads in registers: ReLU, multiply by w, sum (packed f32x2 FMA), scale.
//    The L x L score matrix never leaves the SM.
//  * Streaming top-k: per query a candidate list in shared memory that
//    admits only keys ranked above the query's threshold. In the 64-head
//    configurations (one query per epilogue warpgroup) every warp appends
//    its passing keys with one shared-memory atomic per tile, without a
//    barrier, and candidates are ranked by the composite (score, index) of
//    topk_comp.cuh. The epilogue warps meet only at sync points, scheduled
//    from the fullest list's free room (no list can overflow before the
//    next one); at a sync point where some list is near capacity every
//    warpgroup cuts its list (a sampled threshold, or the exact k-th
//    composite), which raises its threshold. Other configurations keep ascending lists
//    with one warpgroup barrier per tile (ballot + per-warp counts) and
//    block_select cuts. At the end an exact select writes the k winners,
//    -1 padded.
//  * Rows that see no more than k keys select all of them: their work items
//    write 0..t directly and skip the contraction.
//  * Long-row first scheduling: work items (query group, key chunk) are
//    ordered by decreasing length and dealt to persistent CTAs in a snake.
//  * Decode-style calls (one query per sequence) split the key range into
//    chunks whose candidate lists are merged by a second kernel.
//
// Warp roles (one CTA per SM): warp 0 TMA producer, warp 1 MMA issuer,
// warp 2 TMEM allocator, warp 3 idle, warps 4.. epilogue warpgroups.
#pragma once

#include "common.cuh"
#include <type_traits>

#include "topk_comp.cuh"
#include "topk_select.cuh"

// FAST epilogue: of the 8 column pairs of heads a thread reduces per key,
// the first IC_IDX_RELU_REPS take max + packed FMA, the rest the |x| form
// (see the epilogue); 8 keeps every head on the max form.
#ifndef IC_IDX_RELU_REPS
#define IC_IDX_RELU_REPS 8
#endif

namespace ic {

constexpr int IDX_BM = 128;  // keys per tile = MMA M = TMEM lanes

struct IdxParams {
    const void* w;            // [batch, n_q, H_I] bf16 or fp32
    const float* q_scale;     // [batch, n_q] or null
    const float* k_scale;     // [batch, n_k] or null
    int w_is_f32;
    int batch, n_q, n_k, q_pos0, topk;
    int n_groups;             // query groups per batch element
    int n_splits;             // key chunks per group (1 = direct output)
    int chunk;                // keys per chunk (multiple of IDX_BM)
    int n_work;               // n_groups * batch * n_splits
    int32_t* idx_out;         // [batch, n_q, topk]            (n_splits == 1)
    uint32_t* cand_key;       // [batch*n_q, n_splits, topk]   (n_splits > 1)
    int32_t* cand_idx;
    int32_t* cand_cnt;        // [batch*n_q, n_splits]
};

template <int HI_, int G_, int DI_, bool FP8_, int STAGES_, int E_>
struct IdxCfg {
    static constexpr int HI = HI_, G = G_, DI = DI_, STAGES = STAGES_, E = E_;
    static constexpr bool FP8 = FP8_;
    static constexpr int N = G * HI;
    static_assert(N % 16 == 0 && N >= 16 && N <= 256, "MMA N");
    static constexpr int ESZ = FP8 ? 1 : 2;
    static constexpr int ROW_BYTES = DI * ESZ;
    static_assert(ROW_BYTES % 128 == 0, "rows must be whole 128-byte swizzle atoms");
    static constexpr int KATOMS = ROW_BYTES / 128;
    static constexpr int ATOM_ELEMS = 128 / ESZ;
    static constexpr int KSTEPS = ROW_BYTES / 32;  // 32 bytes of K per MMA instruction
    static constexpr int NUM_EPI_WG = G >= 4 ? 4 : (G >= 2 ? 2 : 1);
    static constexpr int QPW = G / NUM_EPI_WG;     // queries per epilogue warpgroup
    static constexpr int COLS_PER_WG = QPW * HI;
    static constexpr int LW = COLS_PER_WG < 64 ? COLS_PER_WG : 64;  // TMEM columns per load
    static_assert(LW % HI == 0 || HI > 64, "load width");
    static constexpr int THREADS = 128 + 128 * NUM_EPI_WG;
    // setmaxnreg split of the launch's registers (65536 / THREADS, in steps of 8):
    // the producer/MMA warpgroup drops to 32, the epilogue warpgroups take the rest
    static constexpr int REGS_LAUNCH = ((65536 / THREADS) / 8) * 8 > 255 ? 248 : ((65536 / THREADS) / 8) * 8;
    static constexpr int REGS_CTRL = 32;
    static constexpr int REGS_EPI_RAW =
        ((REGS_LAUNCH * THREADS - 128 * REGS_CTRL) / (128 * NUM_EPI_WG)) / 8 * 8;
    static constexpr int REGS_EPI = REGS_EPI_RAW > 248 ? 248 : REGS_EPI_RAW;
    static_assert(128 * REGS_CTRL + 128 * NUM_EPI_WG * REGS_EPI <= REGS_LAUNCH * THREADS, "register split");
    static constexpr int C = 128 * E;              // candidate capacity per query
    // 64-head configurations with one query per epilogue warpgroup use the
    // barrier-free append and composite-ranked lists (topk_comp.cuh)
    static constexpr bool FAST = (HI == 64 && QPW == 1);
    static constexpr int PSTEP = 1;                // tiles per append step (generic path)
    static constexpr int RELU_REPS = IC_IDX_RELU_REPS;
    static_assert(RELU_REPS >= 0 && RELU_REPS <= 8, "RELU_REPS");
    // FAST: keys one append step can add to a query's list (one tile); the
    // plan needs topk + 2 steps of room so a cut always leaves a free step
    static constexpr int STEP_KEYS = IDX_BM;
    static constexpr int EPI_THREADS = 128 * NUM_EPI_WG;
    static constexpr int Q_BYTES = N * ROW_BYTES;
    static constexpr int K_BYTES = IDX_BM * ROW_BYTES;
    static constexpr int TMEM_COLS = (2 * N <= 32) ? 32 : (2 * N <= 64) ? 64 : (2 * N <= 128) ? 128
                                                                           : (2 * N <= 256) ? 256 : 512;
    static constexpr uint32_t IDESC = make_idesc(IDX_BM, N, FP8 ? FMT_E4M3 : FMT_BF16,
                                                 FP8 ? FMT_E4M3 : FMT_BF16);
    struct WGState {
        int cnt[2][4][QPW * PSTEP];  // generic: per-step ballot counts (tile, query), by step parity
        int count[2][QPW];      // generic: candidate counts, by tile parity
        uint32_t thr[2][QPW];   // generic: insertion thresholds, by tile parity
        unsigned long long fthr;  // FAST: admission threshold (composite)
        unsigned fcount;        // FAST: candidate count (atomic appends)
    };
    using Scratch = typename std::conditional<FAST, CompScratch<128, E>, SelectScratch<128, E>>::type;
    // shared memory layout (byte offsets)
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_K = OFF_Q + Q_BYTES;
    static constexpr int OFF_CK = OFF_K + STAGES * K_BYTES;
    static constexpr int OFF_CI = OFF_CK + G * C * 4;
    static constexpr int OFF_W = OFF_CI + G * C * 4;
    static constexpr int OFF_SCR = OFF_W + G * HI * 4;
    static constexpr int SCR_BYTES = ((int(sizeof(Scratch)) + 15) / 16) * 16;
    static constexpr int OFF_ST = OFF_SCR + NUM_EPI_WG * SCR_BYTES;
    static constexpr int ST_BYTES = ((int(sizeof(WGState)) + 15) / 16) * 16;
    static constexpr int OFF_BAR = OFF_ST + NUM_EPI_WG * ST_BYTES;
    // mbarrier slots: full[STAGES], empty[STAGES], acc_full[2], acc_empty[2],
    // q_full, q_empty, drain (the abort teardown's MMA drain)
    static constexpr int NUM_BARS = 2 * STAGES + 7;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int SMEM_BYTES = OFF_MISC + 16;
    static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;  // slack for 1024-byte alignment
    static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
};

__device__ __forceinline__ float load_w(const IdxParams& p, int64_t i) {
    if (p.w_is_f32) return static_cast<const float*>(p.w)[i];
    return __bfloat162float(static_cast<const __nv_bfloat16*>(p.w)[i]);
}

struct IdxWork {
    int b, q0, nq_valid, k_begin, k_end, n_tiles;
    bool trivial;  // every query of the group sees at most topk keys: all are selected
};

template <class Cfg>
__device__ __forceinline__ IdxWork idx_work(const IdxParams& p, int item) {
    IdxWork w;
    const int S = p.n_splits;
    const int c = item % S;
    const int rest = item / S;
    w.b = rest % p.batch;
    const int g = p.n_groups - 1 - rest / p.batch;  // longest rows first
    w.q0 = g * Cfg::G;
    w.nq_valid = min(Cfg::G, p.n_q - w.q0);
    const int p_last = p.q_pos0 + w.q0 + w.nq_valid - 1;
    const int n_vis = max(0, min(p_last + 1, p.n_k));
    w.k_begin = c * p.chunk;
    w.k_end = min(n_vis, (c + 1) * p.chunk);
    w.n_tiles = w.k_end > w.k_begin ? ceil_div(w.k_end - w.k_begin, IDX_BM) : 0;
    // the selection of a query that sees at most topk keys is all of them (no
    // scores needed); only for direct output (split chunks feed the merge)
    w.trivial = S == 1 && n_vis <= p.topk;
    if (w.trivial) w.n_tiles = 0;
    return w;
}

__device__ __forceinline__ int snake_item(int round, int cta, int ncta) {
    return round * ncta + ((round & 1) ? (ncta - 1 - cta) : cta);
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
    indexer_topk_kernel(const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k, const IdxParams p) {
    constexpr int HI = Cfg::HI, G = Cfg::G, QPW = Cfg::QPW, E = Cfg::E, C = Cfg::C;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align_smem_1024(smem_raw);
    const uint32_t s_base = smem_u32(smem);
    uint32_t* cand_key_s = reinterpret_cast<uint32_t*>(smem + Cfg::OFF_CK);
    int32_t* cand_idx_s = reinterpret_cast<int32_t*>(smem + Cfg::OFF_CI);
    float* w_s = reinterpret_cast<float*>(smem + Cfg::OFF_W);
    const uint32_t bar0 = s_base + Cfg::OFF_BAR;
    auto bar_full = [&](int s) { return bar0 + 8u * s; };
    auto bar_empty = [&](int s) { return bar0 + 8u * (Cfg::STAGES + s); };
    auto bar_acc_full = [&](int a) { return bar0 + 8u * (2 * Cfg::STAGES + a); };
    auto bar_acc_empty = [&](int a) { return bar0 + 8u * (2 * Cfg::STAGES + 2 + a); };
    const uint32_t bar_q_full = bar0 + 8u * (2 * Cfg::STAGES + 4);
    const uint32_t bar_q_empty = bar0 + 8u * (2 * Cfg::STAGES + 5);
    const uint32_t bar_drain = bar0 + 8u * (2 * Cfg::STAGES + 6);
    static_assert(Cfg::NUM_BARS == 2 * Cfg::STAGES + 7, "barrier slots");
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::OFF_MISC + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < Cfg::STAGES; ++s) {
            mbar_init(bar_full(s), 1);
            mbar_init(bar_empty(s), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(bar_acc_full(a), 1);
            mbar_init(bar_acc_empty(a), 4 * Cfg::NUM_EPI_WG);
        }
        mbar_init(bar_q_full, 1);
        mbar_init(bar_q_empty, 1);
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
    }
    if (warp == 2) {
        tmem_alloc(smem_u32(tmem_slot), Cfg::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int n_rounds = ceil_div(p.n_work, static_cast<int>(gridDim.x));
    // copies issued by the producer: Q loads armed, K tiles armed (counts)
    uint32_t q_armed = 0, k_armed = 0;

    if (warp < 4) {
      regs_dec<Cfg::REGS_CTRL>();
      if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            uint32_t kst = 0, qit = 0;
            int ks_stage = 0;        // kst % STAGES
            uint32_t ks_phase = 0;   // (kst / STAGES) & 1
            for (int r = 0; r < n_rounds; ++r) {
                const int item = snake_item(r, blockIdx.x, gridDim.x);
                if (item >= p.n_work) continue;
                const IdxWork wk = idx_work<Cfg>(p, item);
                if (wk.n_tiles == 0) continue;
                // a wait that fails means the CTA aborted: nothing more is issued
                if (mbar_wait(bar_q_empty, (qit & 1) ^ 1, abort_flag)) {
                    mbar_arrive_expect_tx(bar_q_full, Cfg::Q_BYTES);
                    const int qrow = (wk.b * p.n_q + wk.q0) * HI;
#pragma unroll
                    for (int a = 0; a < Cfg::KATOMS; ++a)
                        tma_load_2d(s_base + Cfg::OFF_Q + a * Cfg::N * 128, &tm_q, bar_q_full,
                                    a * Cfg::ATOM_ELEMS, qrow);
                    q_armed = qit + 1;
                }
                ++qit;
                for (int t = 0; t < wk.n_tiles; ++t) {
                    const int s = ks_stage;
                    if (mbar_wait(bar_empty(s), ks_phase ^ 1, abort_flag)) {
                        mbar_arrive_expect_tx(bar_full(s), Cfg::K_BYTES);
                        const int krow = wk.b * p.n_k + wk.k_begin + t * IDX_BM;
#pragma unroll
                        for (int a = 0; a < Cfg::KATOMS; ++a)
                            tma_load_2d(s_base + Cfg::OFF_K + s * Cfg::K_BYTES + a * IDX_BM * 128, &tm_k,
                                        bar_full(s), a * Cfg::ATOM_ELEMS, krow);
                        k_armed = kst + 1;
                    }
                    ++kst;
                    if (++ks_stage == Cfg::STAGES) {
                        ks_stage = 0;
                        ks_phase ^= 1;
                    }
                }
            }
        }
      } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            uint32_t qit = 0, ait = 0;
            int ks_stage = 0;        // key tile count % STAGES
            uint32_t ks_phase = 0;   // (key tile count / STAGES) & 1
            for (int r = 0; r < n_rounds; ++r) {
                const int item = snake_item(r, blockIdx.x, gridDim.x);
                if (item >= p.n_work) continue;
                const IdxWork wk = idx_work<Cfg>(p, item);
                if (wk.n_tiles == 0) continue;
                mbar_wait(bar_q_full, qit & 1, abort_flag);
                ++qit;
                tc_fence_after();
                for (int t = 0; t < wk.n_tiles; ++t) {
                    const int s = ks_stage;
                    const uint32_t kph = ks_phase;
                    if (++ks_stage == Cfg::STAGES) {
                        ks_stage = 0;
                        ks_phase ^= 1;
                    }
                    const int a = ait & 1;
                    const bool go = mbar_wait(bar_full(s), kph, abort_flag) &&
                                    mbar_wait(bar_acc_empty(a), ((ait >> 1) & 1) ^ 1, abort_flag);
                    tc_fence_after();
                    if (!go) {  // aborted: issue nothing more; the teardown drains
                        ++ait;
                        continue;
                    }
                    const uint32_t d_tmem = tmem_base + a * Cfg::N;
                    const uint64_t adesc0 = make_sw128_desc(s_base + Cfg::OFF_K + s * Cfg::K_BYTES);
                    const uint64_t bdesc0 = make_sw128_desc(s_base + Cfg::OFF_Q);
#pragma unroll
                    for (int ks = 0; ks < Cfg::KSTEPS; ++ks) {
                        const int atom = ks >> 2;
                        const uint32_t koff = (ks & 3) * 32;
                        const uint64_t adesc = adesc0 + ((atom * IDX_BM * 128 + koff) >> 4);
                        const uint64_t bdesc = bdesc0 + ((atom * Cfg::N * 128 + koff) >> 4);
                        if constexpr (Cfg::FP8)
                            mma_f8(d_tmem, adesc, bdesc, Cfg::IDESC, ks > 0 ? 1u : 0u);
                        else
                            mma_f16(d_tmem, adesc, bdesc, Cfg::IDESC, ks > 0 ? 1u : 0u);
                    }
                    mma_commit(bar_empty(s));
                    mma_commit(bar_acc_full(a));
                    ++ait;
                }
                mma_commit(bar_q_empty);
            }
        }
      }
    } else {
        regs_inc<Cfg::REGS_EPI>();
        // ------------------------------------------------------------ epilogue
        const int e = (warp - 4) >> 2;            // epilogue warpgroup
        const int wq = warp & 3;                  // TMEM lane quarter
        const int wtid = threadIdx.x - 128 - 128 * e;
        const int bar_id = 1 + e;
        typename Cfg::Scratch& sc =
            *reinterpret_cast<typename Cfg::Scratch*>(smem + Cfg::OFF_SCR + e * Cfg::SCR_BYTES);
        typename Cfg::WGState& st =
            *reinterpret_cast<typename Cfg::WGState*>(smem + Cfg::OFF_ST + e * Cfg::ST_BYTES);
        uint32_t ait = 0;
        int par = 0;
        for (int r = 0; r < n_rounds; ++r) {
            const int item = snake_item(r, blockIdx.x, gridDim.x);
            if (item >= p.n_work) continue;
            const IdxWork wk = idx_work<Cfg>(p, item);
            const int c_split = item % p.n_splits;
            if (wk.trivial) {
                // every visible key is selected: 0..n_vis-1, then -1 (the index
                // buffer may still be read by the previous kernel of a layer loop)
                griddep_sync();
                for (int gl = 0; gl < QPW; ++gl) {
                    const int g = e * QPW + gl;
                    if (g >= wk.nq_valid) continue;
                    const int64_t row = static_cast<int64_t>(wk.b) * p.n_q + wk.q0 + g;
                    const int n_vis = max(0, min(p.q_pos0 + wk.q0 + g + 1, p.n_k));
                    int32_t* out = p.idx_out + row * p.topk;
                    for (int i = wtid; i < p.topk; i += 128) out[i] = i < n_vis ? i : -1;
                }
                continue;
            }
            // per-query head weights, folded with the query's token scale
            for (int i = wtid; i < Cfg::COLS_PER_WG; i += 128) {
                const int g = e * QPW + i / HI;
                const int j = i % HI;
                float v = 0.f;
                if (g < wk.nq_valid) {
                    const int64_t row = static_cast<int64_t>(wk.b) * p.n_q + wk.q0 + g;
                    v = load_w(p, row * HI + j);
                    if (p.q_scale) v *= p.q_scale[row];
                }
                w_s[g * HI + j] = v;
            }
            if constexpr (Cfg::FAST) {
                if (wtid == 0) {
                    st.fcount = 0u;
                    st.fthr = 0ull;
                }
            } else {
                for (int i = wtid; i < QPW; i += 128) {
                    st.count[par][i] = 0;
                    st.thr[par][i] = 0u;
                }
            }
            named_bar_sync(bar_id, 128);

            // Key owned by this thread after the head reduction. The generic path
            // reads TMEM with the 32x32b shape (thread = lane = key) and every
            // thread reads all head weights. The 64-head path reads the 16x256b
            // shape: a thread holds 16 heads of 4 keys, so it reads only those 16
            // weights, and the 4 threads sharing the keys finish the sum with a
            // reduce-scatter that leaves key r + 8 i(c) in lane 4r + c.
            constexpr bool FAST = Cfg::FAST;
            const int c4 = lane & 3, r8 = lane >> 2;
            const int kidx = FAST ? r8 + 8 * (2 * (c4 & 1) + (c4 >> 1)) : lane;
            // lanes whose key precedes this lane's key (for the in-order append)
            uint32_t rank_mask = 0;
#pragma unroll 1
            for (int l = 0; l < 32; ++l) {
                const int kl = FAST ? (l >> 2) + 8 * (2 * (l & 1) + ((l & 3) >> 1)) : l;
                if (kl < kidx) rank_mask |= 1u << l;
            }
            const int key_lane = wq * 32 + kidx;
            auto key_scale = [&](int t) {
                const int sk = wk.k_begin + t * IDX_BM + key_lane;
                return (p.k_scale != nullptr && t < wk.n_tiles && sk < wk.k_end)
                           ? p.k_scale[static_cast<int64_t>(wk.b) * p.n_k + sk]
                           : 1.f;
            };
            float ksc_next = key_scale(0);

            if constexpr (FAST) {
              // ---------------- 64 heads, one query per warpgroup: barrier-free append
              uint32_t* ck = cand_key_s + e * C;
              int32_t* ci = cand_idx_s + e * C;
              auto load_key = [&](int pos) { return ck[pos]; };
              auto load_id = [&](int pos) { return ci[pos]; };
              auto comp_at = [&](int pos) { return comp_key(ck[pos], ci[pos]); };
              const int pos_g = p.q_pos0 + wk.q0 + e;
              uint64_t thr = 0ull;  // admission threshold; changes only in cuts
              // The epilogue warps meet every `per` tiles. A list that an append
              // left above `hw` since the last meeting makes every warpgroup cut
              // its list there; otherwise every list is at most hw long, and the
              // next `per` tiles (128 keys each) fit: no list ever overflows.
              const int per = (Cfg::C - p.topk >= 10 * IDX_BM) ? 4 : 2;
              const int hw = Cfg::C - per * IDX_BM;
              bool crossed = false;  // lane 0: this warp left its list above hw since the last meeting
              // TMEM -> registers: keys r, r+8 (ra) and r+16, r+24 (rb) of this
              // warp's lane quarter, 16 heads each. The loads of tile t+1 are
              // issued before the append of tile t, so their latency overlaps it.
              uint32_t ra[32], rb[32];
              const uint32_t tb0 = tmem_base + (static_cast<uint32_t>(wq * 32) << 16) + e * Cfg::COLS_PER_WG;
              auto issue_loads = [&](uint32_t it) {
                  mbar_wait(bar_acc_full(it & 1), (it >> 1) & 1, abort_flag);
                  tc_fence_after();
                  const uint32_t tb = tb0 + (it & 1) * Cfg::N;
                  tmem_ld_16x256b_x8(tb, ra);
                  tmem_ld_16x256b_x8(tb + (16u << 16), rb);
              };
              // per-item constants of the tile loop: the last key this lane's
              // query may select (-1: none), the key scales of the batch element
              const int key_hi = e < wk.nq_valid ? min(wk.k_end - 1, pos_g) : -1;
              const float* ks_row = p.k_scale != nullptr ? p.k_scale + static_cast<int64_t>(wk.b) * p.n_k : nullptr;
              auto scale_of = [&](int sk) { return (ks_row != nullptr && sk < wk.k_end) ? ks_row[sk] : 1.f; };
              int s_key = wk.k_begin + key_lane;  // this lane's key in the current tile
              float ksc_f = scale_of(s_key);
              int till_meet = per;
              if (wk.n_tiles > 0) issue_loads(ait);
              // two tiles per loop trip: the loop's bookkeeping is a measurable
              // share of the epilogue's issue slots
#pragma unroll 2
              for (int t = 0; t < wk.n_tiles; ++t, ++ait, s_key += IDX_BM) {
                const int a = ait & 1;
                // the next tile's key scale is requested a whole tile ahead
                const float ksc = ksc_f;
                ksc_f = scale_of(s_key + IDX_BM);
                // this lane's 16 head weights (8-byte loads shared by the 8 lanes
                // of a column pair)
                float2 wreg[8];
                const float* wg = w_s + e * HI + 2 * c4;
#pragma unroll
                for (int i = 0; i < 8; ++i) wreg[i] = *reinterpret_cast<const float2*>(wg + 8 * i);
                tmem_wait_ld();
                // Heads of the first RELU_REPS column pairs: w . ReLU(x) (max on the
                // ALU, packed FMA); the rest: w . ReLU(x) = (w.x + w.|x|) / 2 with |x|
                // an FMA operand, which moves the work to the FMA pipe
                float2 acc[4], lin[4];
                float aab[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    acc[u] = make_float2(0.f, 0.f);
                    lin[u] = make_float2(0.f, 0.f);
                    aab[u] = 0.f;
                }
                auto relu2 = [](uint32_t x, uint32_t y) {
                    return make_float2(fmaxf(__uint_as_float(x), 0.f), fmaxf(__uint_as_float(y), 0.f));
                };
                auto head_pair = [&](int i, uint32_t x, uint32_t y, int u) {
                    if (i < Cfg::RELU_REPS) {
                        acc[u] = __ffma2_rn(wreg[i], relu2(x, y), acc[u]);
                    } else {
                        lin[u] = __ffma2_rn(wreg[i], make_float2(__uint_as_float(x), __uint_as_float(y)), lin[u]);
                        aab[u] = fmaf(wreg[i].x, fabsf(__uint_as_float(x)), aab[u]);
                        aab[u] = fmaf(wreg[i].y, fabsf(__uint_as_float(y)), aab[u]);
                    }
                };
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    head_pair(i, ra[4 * i], ra[4 * i + 1], 0);      // key r
                    head_pair(i, ra[4 * i + 2], ra[4 * i + 3], 1);  // key r + 8
                    head_pair(i, rb[4 * i], rb[4 * i + 1], 2);      // key r + 16
                    head_pair(i, rb[4 * i + 2], rb[4 * i + 3], 3);  // key r + 24
                }
                // the accumulator stage is free once read
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_acc_empty(a));
                // every `per` tiles, except after the last: the same in every epilogue thread
                const bool meet = --till_meet == 0 && t + 1 < wk.n_tiles;
                if (till_meet == 0) till_meet = per;
                float pk[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    pk[u] = acc[u].x + acc[u].y;
                    if (Cfg::RELU_REPS < 8) pk[u] += 0.5f * ((lin[u].x + lin[u].y) + aab[u]);
                }
                // reduce-scatter over the 4 lanes of a row: after the xor-1 step a
                // lane holds keys {0,1} (even c) or {2,3} (odd c) of its row, after
                // the xor-2 step one key
                const bool odd = (c4 & 1) != 0;
                const float q0 = (odd ? pk[2] : pk[0]) + __shfl_xor_sync(0xffffffffu, odd ? pk[0] : pk[2], 1);
                const float q1 = (odd ? pk[3] : pk[1]) + __shfl_xor_sync(0xffffffffu, odd ? pk[1] : pk[3], 1);
                const bool hi2 = (c4 & 2) != 0;
                const float sum = (hi2 ? q1 : q0) + __shfl_xor_sync(0xffffffffu, hi2 ? q0 : q1, 2);
                const uint32_t kk = float_to_ordered(sum * ksc);
                const bool valid = s_key <= key_hi;

                // ---- append this tile's passing keys (one atomic per warp)
                const bool pass = valid && comp_key(kk, s_key) > thr;
                const uint32_t bal = __ballot_sync(0xffffffffu, pass);
                if (bal != 0u) {
                    unsigned base = 0u;
                    if (lane == 0) {
                        const unsigned nb = static_cast<unsigned>(__popc(bal));
                        base = atomicAdd(&st.fcount, nb);
                        crossed |= base + nb > static_cast<unsigned>(hw);
                    }
                    base = __shfl_sync(0xffffffffu, base, 0);
                    if (pass) {
                        const int pos = static_cast<int>(base) + __popc(bal & rank_mask);
                        if (IC_DCHECK(pos < C)) {
                            ck[pos] = kk;
                            ci[pos] = s_key;
                        }
                    }
                }

                // the next tile's TMEM loads go out after the append (issued before
                // it, they measured ~500 cycles per tile slower)
                if (!meet && t + 1 < wk.n_tiles) issue_loads(ait + 1);
                if (meet) {
                    // ---- meeting: every list's appends so far are done; the OR says
                    // whether any list passed hw
                    const bool any = named_bar_or(5, Cfg::EPI_THREADS, crossed);
                    crossed = false;
                    if (any) {
                        // every list past the middle of [topk, hw] is cut to its exact
                        // top-k at this tile (the warpgroups stall together); a list
                        // left uncut stays below hw
                        const int n = static_cast<int>(st.fcount);  // same in the whole warpgroup
                        if (n > (p.topk + hw) / 2) {
                            const uint64_t tau =
                                comp_select_kth<128, E>(n, p.topk, wtid, bar_id, sc, load_key, load_id);
                            const int kept = comp_compact<128, E>(
                                n, wtid, bar_id, sc, load_key, load_id, [&](int pos) { return comp_at(pos) >= tau; },
                                [&](int o, uint32_t kv, int32_t iv) {
                                    if (IC_DCHECK(o < n)) {
                                        ck[o] = kv;
                                        ci[o] = iv;
                                    }
                                });
                            // no key ranked below tau can win: k kept keys rank at or above it
                            if (wtid == 0) {
                                st.fcount = static_cast<unsigned>(kept);
                                st.fthr = tau;
                            }
                            named_bar_sync(bar_id, 128);
                            thr = st.fthr;
                        }
                    }
                    issue_loads(ait + 1);
                }
              }
              // every warp's appends must be visible to the final select; the
              // outputs may still be read by the previous kernel of a layer loop
              griddep_sync();
              named_bar_sync(bar_id, 128);
              if (e < wk.nq_valid) {  // uniform across the warpgroup
                  const int n = static_cast<int>(st.fcount);
                  const int64_t row = static_cast<int64_t>(wk.b) * p.n_q + wk.q0 + e;
                  uint64_t tau = 0ull;
                  if (n > p.topk) tau = comp_select_kth<128, E>(n, p.topk, wtid, bar_id, sc, load_key, load_id);
                  auto keep = [&](int pos) { return comp_at(pos) >= tau; };
                  // warp wq appended keys with (s mod 128) in [32 wq, 32 wq + 32), in
                  // ascending order: group-major emission is deterministic
                  auto group = [&](int pos) { return (ci[pos] & (IDX_BM - 1)) >> 5; };
                  if (p.n_splits == 1) {
                      int32_t* out = p.idx_out + row * p.topk;
                      const int kept = comp_emit_grouped<128, E>(n, wtid, bar_id, sc, keep, group, [&](int o, int pos) {
                          if (IC_DCHECK(o < p.topk)) out[o] = ci[pos];
                      });
                      for (int i = kept + wtid; i < p.topk; i += 128) out[i] = -1;
                  } else {
                      const int64_t slot = row * p.n_splits + c_split;
                      uint32_t* okey = p.cand_key + slot * p.topk;
                      int32_t* oidx = p.cand_idx + slot * p.topk;
                      const int kept = comp_emit_grouped<128, E>(n, wtid, bar_id, sc, keep, group,
                                                                 [&](int o, int pos) {
                                                                     if (IC_DCHECK(o < p.topk)) {
                                                                         okey[o] = ck[pos];
                                                                         oidx[o] = ci[pos];
                                                                     }
                                                                 });
                      if (wtid == 0) p.cand_cnt[slot] = kept;
                  }
              }
              named_bar_sync(bar_id, 128);
            } else {
            constexpr int PS = Cfg::PSTEP;
            for (int t = 0; t < wk.n_tiles; t += PS) {
              // score PS tiles (releasing each accumulator stage as soon as it is
              // read), then one barrier and one append step for all of them
              uint32_t keyv[QPW * PS];
              uint32_t passmask = 0;
              int skey[PS];
#pragma unroll
              for (int sub = 0; sub < PS; ++sub) {
                const int tt = t + sub;
                skey[sub] = wk.k_begin + tt * IDX_BM + key_lane;
#pragma unroll
                for (int gl = 0; gl < QPW; ++gl) keyv[sub * QPW + gl] = 0u;
                if (tt >= wk.n_tiles) continue;  // uniform across the warpgroup
                const int a = ait & 1;
                // the next tile's key scale is requested a whole tile ahead
                const float ksc = ksc_next;
                ksc_next = key_scale(tt + 1);
                mbar_wait(bar_acc_full(a), (ait >> 1) & 1, abort_flag);
                tc_fence_after();
                const int s_key = skey[sub];
                const bool in_range = s_key < wk.k_end;
                const uint32_t taddr =
                    tmem_base + (static_cast<uint32_t>(wq * 32) << 16) + a * Cfg::N + e * Cfg::COLS_PER_WG;
#pragma unroll
                for (int c0 = 0; c0 < Cfg::COLS_PER_WG; c0 += Cfg::LW) {
                    uint32_t regs[Cfg::LW];
                    tmem_ld<Cfg::LW>(taddr + c0, regs);
                    tmem_wait_ld();
#pragma unroll
                    for (int qq = 0; qq < Cfg::LW / HI; ++qq) {
                        const int gl = c0 / HI + qq;
                        const int g = e * QPW + gl;
                        const float* wg = w_s + g * HI;
                        // four independent packed accumulators keep the FMA chains short
                        constexpr int NACC = HI >= 16 ? 4 : HI / 4 > 0 ? HI / 4 : 1;
                        float2 acc[2 * NACC];
#pragma unroll
                        for (int a2 = 0; a2 < 2 * NACC; ++a2) acc[a2] = make_float2(0.f, 0.f);
#pragma unroll
                        for (int j = 0; j < HI; j += 4) {
                            const float4 w4 = *reinterpret_cast<const float4*>(wg + j);
                            const float x0 = fmaxf(__uint_as_float(regs[qq * HI + j + 0]), 0.f);
                            const float x1 = fmaxf(__uint_as_float(regs[qq * HI + j + 1]), 0.f);
                            const float x2 = fmaxf(__uint_as_float(regs[qq * HI + j + 2]), 0.f);
                            const float x3 = fmaxf(__uint_as_float(regs[qq * HI + j + 3]), 0.f);
                            const int slot = (j / 4) % NACC;
                            acc[2 * slot] = __ffma2_rn(make_float2(w4.x, w4.y), make_float2(x0, x1), acc[2 * slot]);
                            acc[2 * slot + 1] =
                                __ffma2_rn(make_float2(w4.z, w4.w), make_float2(x2, x3), acc[2 * slot + 1]);
                        }
#pragma unroll
                        for (int a2 = 2 * NACC / 2; a2 >= 1; a2 /= 2) {
#pragma unroll
                            for (int b2 = 0; b2 < a2; ++b2) acc[b2] = __fadd2_rn(acc[b2], acc[b2 + a2]);
                        }
                        const float score = (acc[0].x + acc[0].y) * ksc;
                        const uint32_t kk = float_to_ordered(score);
                        const int pos_g = p.q_pos0 + wk.q0 + g;
                        const bool valid = in_range && g < wk.nq_valid && s_key <= pos_g;
                        keyv[sub * QPW + gl] = kk;
                        if (valid && kk > st.thr[par][gl]) passmask |= 1u << (sub * QPW + gl);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_acc_empty(a));
                ++ait;
              }
              uint32_t bal[QPW * PS];
#pragma unroll
              for (int j = 0; j < QPW * PS; ++j) {
                  bal[j] = __ballot_sync(0xffffffffu, (passmask >> j) & 1u);
                  if (lane == 0) st.cnt[par][wq][j] = __popc(bal[j]);
              }
              named_bar_sync(bar_id, 128);
#pragma unroll 1
              for (int gl = 0; gl < QPW; ++gl) {
                  const int g = e * QPW + gl;
                  int tot[PS], before[PS], total = 0;
#pragma unroll
                  for (int sub = 0; sub < PS; ++sub) {
                      tot[sub] = 0;
                      before[sub] = 0;
#pragma unroll
                      for (int w4 = 0; w4 < 4; ++w4) {
                          const int cw = st.cnt[par][w4][sub * QPW + gl];
                          tot[sub] += cw;
                          if (w4 < wq) before[sub] += cw;
                      }
                      total += tot[sub];
                  }
                  int cnt_g = st.count[par][gl];
                  uint32_t thr_g = st.thr[par][gl];
                  uint32_t* ck = cand_key_s + g * C;
                  int32_t* ci = cand_idx_s + g * C;
                  if (cnt_g + total > C) {
                      // cut the list back and raise the threshold
                      bool cut = false;
                      if (C - p.topk >= 1536) {
                          // sampled cut: 32 keys spread over the list, sorted by one
                          // warp, give tau with ~ k + 2 sigma of the list above it; the
                          // keys above tau are compacted in place when there are
                          // between k and C - (one step) of them (none can be a
                          // winner otherwise lost: at least k kept keys beat them)
                          if (wq == 0) {
                              const int pos = static_cast<int>((static_cast<int64_t>(2 * lane + 1) * cnt_g) / 64);
                              uint32_t sk = ck[pos];
                              int sp = pos;
                              warp_sort_desc(sk, sp, lane);
                              const int target = p.topk + (C - p.topk) / 3;
                              const int r = min(31, max(0, (32 * target) / cnt_g));
                              const uint32_t tau_w = __shfl_sync(0xffffffffu, sk, r);
                              if (lane == 0) sc.misc[7] = static_cast<int>(tau_w);
                          }
                          named_bar_sync(bar_id, 128);
                          const uint32_t tau = static_cast<uint32_t>(sc.misc[7]);
                          const int hi = C - IDX_BM * PS;
                          const int kept = block_compact<128, E>(
                              cnt_g, wtid, bar_id, sc, [&](int pos) { return ck[pos]; },
                              [&](int pos) { return ci[pos]; }, [&](uint32_t k) { return k > tau; },
                              [&](int c) { return c >= p.topk && c <= hi; },
                              [&](int pos, uint32_t kv, int32_t iv) {
                                  if (IC_DCHECK(pos < C)) {
                                      ck[pos] = kv;
                                      ci[pos] = iv;
                                  }
                              });
                          if (kept >= 0) {
                              cnt_g = kept;
                              thr_g = max(thr_g, tau);
                              cut = true;
                          }
                      }
                      if (!cut) {
                          const int relax = max(p.topk, min((p.topk + C) / 2, C - IDX_BM * PS));
                          const SelectResult sr = block_select<128, E>(
                              cnt_g, p.topk, false, relax, thr_g, wtid, bar_id, sc,
                              [&](int pos) { return ck[pos]; }, [&](int pos) { return ci[pos]; },
                              [&](int pos, uint32_t kv, int32_t iv) {
                                  if (IC_DCHECK(pos < C)) {
                                      ck[pos] = kv;
                                      ci[pos] = iv;
                                  }
                              });
                          cnt_g = sr.kept;
                          thr_g = sr.thr;
                      }
                  }
                  int run = cnt_g;
#pragma unroll
                  for (int sub = 0; sub < PS; ++sub) {
                      const int j = sub * QPW + gl;
                      if ((passmask >> j) & 1u) {
                          uint32_t my_key = 0;
#pragma unroll
                          for (int q = 0; q < QPW * PS; ++q)
                              if (q == j) my_key = keyv[q];
                          const int pos = run + before[sub] + __popc(bal[j] & rank_mask);
                          if (IC_DCHECK(pos < C)) {
                              ck[pos] = my_key;
                              ci[pos] = skey[sub];
                          }
                      }
                      run += tot[sub];
                  }
                  // every thread holds the same values: each writes them, so each
                  // later reads its own write and no barrier is needed here
                  st.count[par ^ 1][gl] = cnt_g + total;
                  st.thr[par ^ 1][gl] = thr_g;
              }
              par ^= 1;
            }
            // candidates appended by the other warps must be visible to the final
            // select; the outputs may still be read by the previous kernel
            griddep_sync();
            named_bar_sync(bar_id, 128);

            // ---- final exact selection for each query of this warpgroup
#pragma unroll 1
            for (int gl = 0; gl < QPW; ++gl) {
                const int g = e * QPW + gl;
                if (g >= wk.nq_valid) continue;  // uniform across the warpgroup
                const int n = st.count[par][gl];
                const uint32_t* ck = cand_key_s + g * C;
                const int32_t* ci = cand_idx_s + g * C;
                auto load_key = [&](int pos) { return ck[pos]; };
                auto load_id = [&](int pos) { return ci[pos]; };
                const int64_t row = static_cast<int64_t>(wk.b) * p.n_q + wk.q0 + g;
                if (p.n_splits == 1) {
                    int32_t* out = p.idx_out + row * p.topk;
                    const SelectResult sr = block_select<128, E>(
                        n, p.topk, true, p.topk, 0u, wtid, bar_id, sc, load_key, load_id,
                        [&](int pos, uint32_t, int32_t iv) {
                            if (IC_DCHECK(pos < p.topk)) out[pos] = iv;
                        });
                    for (int i = sr.kept + wtid; i < p.topk; i += 128) out[i] = -1;
                } else {
                    const int64_t slot = row * p.n_splits + c_split;
                    uint32_t* ok = p.cand_key + slot * p.topk;
                    int32_t* oi = p.cand_idx + slot * p.topk;
                    const SelectResult sr = block_select<128, E>(
                        n, p.topk, true, p.topk, 0u, wtid, bar_id, sc, load_key, load_id,
                        [&](int pos, uint32_t kv, int32_t iv) {
                            if (IC_DCHECK(pos < p.topk)) {
                                ok[pos] = kv;
                                oi[pos] = iv;
                            }
                        });
                    if (wtid == 0) p.cand_cnt[slot] = sr.kept;
                }
            }
            named_bar_sync(bar_id, 128);
            }  // generic path
        }
    }

    // ---------------------------------------------------------------- teardown
    __syncthreads();
    if (*abort_flag) {  // final after the barrier: the same in every thread
        // let the copies and MMAs issued before the abort land before the
        // shared and tensor memory they write goes away
        if (warp == 0 && lane == 0) {
            if (q_armed > 0) mbar_drain(bar_q_full, (q_armed - 1) & 1);
            for (uint32_t i = k_armed > Cfg::STAGES ? k_armed - Cfg::STAGES : 0; i < k_armed; ++i)
                mbar_drain(bar_full(i % Cfg::STAGES), (i / Cfg::STAGES) & 1);
        }
        if (warp == 1 && lane == 0) {
            mma_commit(bar_drain);
            mbar_drain(bar_drain, 0);
        }
        __syncthreads();
    }
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
    }
}

// Merge the per-chunk candidate lists of one query row into its final top-k
// (used when the key range was split). One 256-thread CTA per row. The lists
// are copied into shared memory one after the other (dynamic: 8 bytes per
// candidate, 256 * E candidates at most); candidates are ranked by their
// composite (score, index), so the order inside each list does not matter,
// and the winners are written in the (deterministic) concatenated order.
template <int E>
__global__ void __launch_bounds__(256)
    topk_merge_kernel(const uint32_t* __restrict__ cand_key, const int32_t* __restrict__ cand_idx,
                      const int32_t* __restrict__ cand_cnt, int n_splits, int topk,
                      int32_t* __restrict__ idx_out) {
    __shared__ CompScratch<256, E> sc;
    __shared__ int offs[17];
    extern __shared__ uint32_t merge_smem[];
    uint32_t* mkey = merge_smem;
    int32_t* midx = reinterpret_cast<int32_t*>(merge_smem + 256 * E);
    const int row = blockIdx.x;
    const int tid = threadIdx.x;
    griddep_sync();  // the candidate lists come from the previous kernel
    if (tid == 0) {
        int o = 0;
        for (int c = 0; c < n_splits; ++c) {
            offs[c] = o;
            int cnt = cand_cnt[static_cast<int64_t>(row) * n_splits + c];
            if (!in_bounds(cnt >= 0 && cnt <= topk && o + cnt <= 256 * E)) cnt = 0;
            o += cnt;
        }
        offs[n_splits] = o;
    }
    __syncthreads();
    for (int c = 0; c < n_splits; ++c) {
        const int64_t src = (static_cast<int64_t>(row) * n_splits + c) * topk;
        const int cnt = offs[c + 1] - offs[c];
        for (int i = tid; i < cnt; i += 256) {
            mkey[offs[c] + i] = cand_key[src + i];
            midx[offs[c] + i] = cand_idx[src + i];
        }
    }
    __syncthreads();
    const int n = offs[n_splits];
    int32_t* out = idx_out + static_cast<int64_t>(row) * topk;
    auto load_key = [&](int pos) { return mkey[pos]; };
    auto load_id = [&](int pos) { return midx[pos]; };
    uint64_t tau = 0ull;
    if (n > topk) tau = comp_select_kth<256, E>(n, topk, tid, 1, sc, load_key, load_id);
    const int kept = comp_compact<256, E>(
        n, tid, 1, sc, load_key, load_id, [&](int pos) { return comp_key(mkey[pos], midx[pos]) >= tau; },
        [&](int o, uint32_t, int32_t iv) {
            if (IC_DCHECK(o < topk)) out[o] = iv;
        });
    for (int i = kept + tid; i < topk; i += 256) out[i] = -1;
}

}  // namespace ic
