// Sparse attention over the selected latent-KV rows, for sm_100a.
//
// What it computes (IndexCache paper, Abstract: core attention over the k
// tokens the indexer selected, O(Lk) instead of O(L^2)): for every query row
// and head h,
//     out[h,:] = sum_{s in idx} softmax_s(sm_scale * q[h,:d_qk] . kv[s,:d_qk]) * kv[s,:d_v]
// with all heads sharing the gathered kv rows (MQA-style latent KV).
//
// Mapping to Blackwell (one query row per CTA iteration, persistent CTAs):
//  * The selected rows are gathered 64 at a time into a 128-byte-swizzled
//    tile (one tile = 64 keys x d_qk), double-buffered. Two copy paths run in
//    parallel: TMA row gathers (tile::gather4, four rows x one 128-byte column
//    box per instruction) for the first chunks of each row, 16-byte cp.async
//    from the producer warps for the rest.
//  * Scores are formed transposed, S^T = K_sel . Q^T (tcgen05, M = 64 keys,
//    N = 64 heads, K = d_qk, accumulator in TMEM): each softmax thread then
//    owns one key and holds all its heads in registers.
//  * Softmax uses a fixed per-head reference value m (the first selected
//    key's logit): p = 2^(z - m). Because the reference is fixed, the running
//    output needs no per-tile rescaling; only if some logit exceeds the
//    reference by more than IC_ATTN_RESCALE_LOG2 (a rare, data-dependent
//    event) is the reference raised and the TMEM accumulator rescaled once.
//    The row sum l is accumulated per thread and reduced at the end.
//  * P^T (bf16, keys x heads) is written into the tile's rope columns, which
//    the score MMA no longer needs, and O^T = V^T . P^T runs on tcgen05 with
//    M = 128 rows of d_v (full-rate M), N = 64 heads, both operands read
//    MN-major from the same gathered tile, accumulating in TMEM.
//  * Decode-style calls (few query rows) split each row's selected keys
//    across CTAs; partial (m, l, O) triples are merged by a second kernel.
//
// Warp roles: warps 0-7 softmax / output in two warpgroups, one per half of
// the heads (warp w reads TMEM lane quarter w % 4); warp 12 MMA issuer and
// TMEM owner; warps 8-11 and 13-15 index-row compaction and gather producers
// (TMA + cp.async).
#pragma once

#include "common.cuh"

// Gather split: the first IC_ATTN_TMA_CHUNKS 64-column chunks of every
// selected row come in by TMA row gathers, the rest by cp.async from the
// producer warps; the two copy paths run in parallel.
#ifndef IC_ATTN_TMA_CHUNKS
#define IC_ATTN_TMA_CHUNKS 0
#endif

#ifndef IC_ATTN_RESCALE_LOG2
#define IC_ATTN_RESCALE_LOG2 64.0f
#endif

namespace ic {

struct AttnParams {
    const __nv_bfloat16* kv;   // [batch, n_k, d_qk]
    const int32_t* idx;        // [batch, n_q, topk]
    __nv_bfloat16* out;        // [batch, n_q, H, d_v]            (n_splits == 1)
    float* o_part;             // [rows, n_splits, H, d_v]        (n_splits > 1)
    float* ml_part;            // [rows, n_splits, 2, 64]: m (log2 units), l
    int batch, n_q, n_k, H, topk;
    float sm_scale_log2;       // sm_scale * log2(e)
    int n_splits;
    int n_work;                // rows * n_splits
};

template <int DQK_, int DV_>
struct AttnCfg {
    static constexpr int DQK = DQK_, DV = DV_;
    static_assert(DQK % 64 == 0 && DQK <= 576, "d_qk");
    static_assert(DV % 64 == 0 && DV <= 512 && DV <= DQK, "d_v");
    static_assert(DV % 128 == 0 || DV == 64, "d_v blocks");
    static constexpr int BK = 64;                 // keys per tile (MMA M of S^T)
    static constexpr int NH = 64;                 // padded heads (MMA N)
    static constexpr int NCH = DQK / 64;          // 128-byte column chunks per row
    static constexpr int CH_BYTES = BK * 128;     // one chunk of a tile
    static constexpr bool P_IN_ROPE = DQK > DV;   // P^T reuses the first non-value chunk
    static constexpr int P_CHUNK = P_IN_ROPE ? DV / 64 : NCH;
    static constexpr int TILE_CHUNKS = P_IN_ROPE ? NCH : NCH + 1;
    static constexpr int TILE_BYTES = TILE_CHUNKS * CH_BYTES;
    static constexpr int Q_CH_BYTES = NH * 128;
    static constexpr int Q_BYTES = NCH * Q_CH_BYTES;
    static constexpr int VB_M = DV >= 128 ? 128 : 64;   // rows of d_v per PV MMA
    static constexpr int NVB = DV / VB_M;
    static constexpr int MAX_TOPK = 2048;
    // two softmax warpgroups (warps 0-7), a producer warpgroup (8-11) and a
    // warpgroup of the MMA warp (12) plus three more producers (13-15)
    static constexpr int THREADS = 512;
    static constexpr int MMA_WARP = 12;
    static constexpr int NPROD = 7 * 32;
    static constexpr int SMX_HEADS = NH / 2;  // heads per softmax warpgroup
    // register split after setmaxnreg (launch: 65536 / THREADS = 128 per thread)
    static constexpr int REGS_SOFTMAX = 160, REGS_OTHER = 96;
    static_assert(256 * REGS_SOFTMAX + 256 * REGS_OTHER <= 65536, "register split");
    static constexpr int TMA_CH = IC_ATTN_TMA_CHUNKS < NCH ? IC_ATTN_TMA_CHUNKS : NCH;
    static constexpr uint32_t TILE_TX = BK * TMA_CH * 128;  // bytes gathered by TMA per tile
    static constexpr int KV_FULL_COUNT = (TMA_CH > 0 ? 1 : 0) + (TMA_CH < NCH ? NPROD : 0);
    static constexpr uint32_t IDESC_S = make_idesc(BK, NH, FMT_BF16, FMT_BF16);
    static constexpr uint32_t IDESC_O = make_idesc(VB_M, NH, FMT_BF16, FMT_BF16, 1, 1);
    static constexpr int S_COL = 0;      // S^T buffers at columns [0,64) and [64,128)
    static constexpr int O_COL = 128;    // O^T blocks at 128 + 64*vb
    static constexpr int TMEM_COLS = 512;
    // shared memory layout
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_T = OFF_Q + Q_BYTES;
    static constexpr int OFF_LIST = OFF_T + 2 * TILE_BYTES;
    static constexpr int OFF_M = OFF_LIST + MAX_TOPK * 4;
    static constexpr int OFF_A = OFF_M + 64 * 4;
    static constexpr int OFF_RED = OFF_A + 64 * 4;          // [4][64] floats
    static constexpr int OFF_CNT = OFF_RED + 4 * 64 * 4;    // compaction table [32][2] + misc
    static constexpr int OFF_BAR = OFF_CNT + 80 * 4;
    // mbarrier slots: q_full, q_empty, kv_full[2], kv_empty[2], s_full[2],
    // s_free[2], p_full[2], pv_done, o_free, drain (the abort teardown's MMA drain)
    static constexpr int NUM_BARS = 15;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;
    static constexpr int SMEM_BYTES = OFF_MISC + 32;
    static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;
    static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
};


__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
                 "r"(d)
                 : "memory");
}



struct AttnWork {
    int64_t row;
    int split;
};

__device__ __forceinline__ AttnWork attn_work(const AttnParams& p, int item) {
    AttnWork w;
    const int64_t rows = static_cast<int64_t>(p.batch) * p.n_q;
    w.split = item % p.n_splits;
    w.row = rows - 1 - item / p.n_splits;  // later rows (more keys) first
    return w;
}

__device__ __forceinline__ int attn_snake(int round, int cta, int ncta) {
    return round * ncta + ((round & 1) ? (ncta - 1 - cta) : cta);
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
    sparse_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kv,
                       const AttnParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    const uint32_t s_base = smem_u32(smem);
    int32_t* list_s = reinterpret_cast<int32_t*>(smem + Cfg::OFF_LIST);
    float* m_s = reinterpret_cast<float*>(smem + Cfg::OFF_M);
    float* a_s = reinterpret_cast<float*>(smem + Cfg::OFF_A);
    float* red_s = reinterpret_cast<float*>(smem + Cfg::OFF_RED);
    int* cnt_s = reinterpret_cast<int*>(smem + Cfg::OFF_CNT);
    const uint32_t bar0 = s_base + Cfg::OFF_BAR;
    const uint32_t bar_q_full = bar0 + 0, bar_q_empty = bar0 + 8;
    auto bar_kv_full = [&](int s) { return bar0 + 16u + 8u * s; };
    auto bar_kv_empty = [&](int s) { return bar0 + 32u + 8u * s; };
    auto bar_s_full = [&](int s) { return bar0 + 48u + 8u * s; };
    auto bar_s_free = [&](int s) { return bar0 + 64u + 8u * s; };
    auto bar_p_full = [&](int s) { return bar0 + 80u + 8u * s; };
    const uint32_t bar_pv_done = bar0 + 96, bar_o_free = bar0 + 104, bar_drain = bar0 + 112;
    static_assert(Cfg::NUM_BARS * 8 == 120, "barrier slots end where the misc words begin");
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::OFF_MISC);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::OFF_MISC + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // Q rows past H are never written by the Q copy: zero the buffer once.
    for (int i = threadIdx.x; i < Cfg::Q_BYTES / 16; i += blockDim.x)
        reinterpret_cast<uint4*>(smem + Cfg::OFF_Q)[i] = make_uint4(0, 0, 0, 0);
    if (threadIdx.x == 0) {
        mbar_init(bar_q_full, 1);
        mbar_init(bar_q_empty, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar_kv_full(s), Cfg::KV_FULL_COUNT);
            mbar_init(bar_kv_empty(s), 1);
            mbar_init(bar_s_full(s), 1);
            mbar_init(bar_s_free(s), 8);
            mbar_init(bar_p_full(s), 8);
        }
        mbar_init(bar_pv_done, 1);
        mbar_init(bar_o_free, 8);
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    constexpr int MMA_WARP = Cfg::MMA_WARP;
    if (warp == MMA_WARP) {
        tmem_alloc(smem_u32(tmem_slot), Cfg::TMEM_COLS);
        tmem_relinquish();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // the index rows may come from the previous kernel of a layer loop, and the
    // outputs or partials may still be read by it
    griddep_sync();
    const int n_rounds = ceil_div(p.n_work, static_cast<int>(gridDim.x));
    // copies issued by the producers' first thread: Q loads and KV tiles armed (counts)
    uint32_t q_armed = 0, kv_armed = 0;

    if (warp >= 8) {
      regs_dec<Cfg::REGS_OTHER>();
      if (warp != MMA_WARP) {
        // --------------------------- index compaction + TMA / cp.async row gathers
        const int pw = warp < MMA_WARP ? warp - 8 : warp - 9;  // producer warp 0..6
        const int ptid = pw * 32 + lane;
        if (ptid == 0) {
            prefetch_tmap(&tm_q);
            prefetch_tmap(&tm_kv);
        }
        uint32_t kv_n = 0, q_n = 0;
        for (int r = 0; r < n_rounds; ++r) {
            const int item = attn_snake(r, blockIdx.x, gridDim.x);
            if (item >= p.n_work) continue;
            const AttnWork wk = attn_work(p, item);
            const int b = static_cast<int>(wk.row / p.n_q);
            // compact the valid entries of the index row, keeping their order:
            // producer warp w takes a contiguous segment (all of its loads in
            // flight at once), then the segment counts give the write offsets
            const int32_t* irow = p.idx + wk.row * p.topk;
            constexpr int NPW = Cfg::NPROD / 32;
            constexpr int VPL = (Cfg::MAX_TOPK + NPW * 32 - 1) / (NPW * 32);  // entries per lane
            const int seg = ceil_div(ceil_div(p.topk, NPW), 32) * 32;
            const int e0 = pw * seg;
            int v[VPL];
            int my_cnt = 0;
#pragma unroll
            for (int u = 0; u < VPL; ++u) {
                const int e = e0 + 32 * u + lane;
                v[u] = (32 * u < seg && e < p.topk) ? irow[e] : -1;
                my_cnt += (v[u] >= 0 && v[u] < p.n_k) ? 1 : 0;
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) my_cnt += __shfl_xor_sync(0xffffffffu, my_cnt, o);
            if (lane == 0) cnt_s[1 + pw] = my_cnt;
            named_bar_sync(3, Cfg::NPROD);
            int run = 0, n_total = 0;
#pragma unroll
            for (int w = 0; w < NPW; ++w) {
                const int c = cnt_s[1 + w];
                run += w < pw ? c : 0;
                n_total += c;
            }
#pragma unroll
            for (int u = 0; u < VPL; ++u) {
                const bool ok = v[u] >= 0 && v[u] < p.n_k;
                const uint32_t bal = __ballot_sync(0xffffffffu, ok);
                if (ok) {
                    const int slot = run + __popc(bal & lanemask_lt());
                    if (IC_DCHECK(slot < Cfg::MAX_TOPK)) list_s[slot] = v[u];
                }
                run += __popc(bal);
            }
            if (pw == 0 && lane == 0) cnt_s[0] = n_total;
            named_bar_sync(3, Cfg::NPROD);
            const int n_valid = cnt_s[0];
            const int len = ceil_div(ceil_div(n_valid, p.n_splits), Cfg::BK) * Cfg::BK;
            const int lo = min(n_valid, wk.split * len);
            const int hi = min(n_valid, lo + len);
            const int n_tiles = ceil_div(hi - lo, Cfg::BK);
            if (n_tiles > 0) {
                if (ptid == 0) {
                    // a wait that fails means the CTA aborted: nothing more is issued
                    if (mbar_wait(bar_q_empty, (q_n & 1) ^ 1, abort_flag)) {
                        mbar_arrive_expect_tx(bar_q_full, Cfg::NCH * p.H * 128);
                        const int qrow = static_cast<int>(wk.row) * p.H;
                        for (int a = 0; a < Cfg::NCH; ++a)
                            tma_load_2d(s_base + Cfg::OFF_Q + a * Cfg::Q_CH_BYTES, &tm_q, bar_q_full, a * 64,
                                        qrow);
                        q_armed = q_n + 1;
                    }
                }
                const int row_base = b * p.n_k;
                const int fallback = list_s[lo];  // rows past the slice end re-read a valid row
                const __nv_bfloat16* kvb = p.kv + static_cast<int64_t>(row_base) * Cfg::DQK;
                for (int j = 0; j < n_tiles; ++j) {
                    const int s = kv_n & 1;
                    const bool issue = mbar_wait(bar_kv_empty(s), ((kv_n >> 1) & 1) ^ 1, abort_flag);
                    const uint32_t tile = s_base + Cfg::OFF_T + s * Cfg::TILE_BYTES;
                    if constexpr (Cfg::TMA_CH > 0) {
                        if (ptid == 0 && issue) {
                            kv_armed = kv_n + 1;
                            mbar_arrive_expect_tx(bar_kv_full(s), Cfg::TILE_TX);
                            for (int g = 0; g < Cfg::BK / 4; ++g) {
                                int rows[4];
#pragma unroll
                                for (int i = 0; i < 4; ++i) {
                                    const int e = lo + j * Cfg::BK + 4 * g + i;
                                    rows[i] = row_base + (e < hi ? list_s[e] : fallback);
                                }
                                const uint32_t dst = tile + (g >> 1) * 1024 + (g & 1) * 512;
#pragma unroll
                                for (int a = 0; a < Cfg::TMA_CH; ++a)
                                    tma_gather4(dst + a * Cfg::CH_BYTES, &tm_kv, bar_kv_full(s), a * 64,
                                                rows[0], rows[1], rows[2], rows[3]);
                            }
                        }
                    }
                    if (Cfg::TMA_CH < Cfg::NCH && issue) {
                        // cp.async for chunks [TMA_CH, NCH): warp pw takes rows pw, pw+NW, ...
                        constexpr int NW = Cfg::NPROD / 32;
                        constexpr int UPR = (Cfg::NCH - Cfg::TMA_CH) * 8;  // 16-byte units per row
                        constexpr int UPL = (UPR + 31) / 32;
                        for (int rr = pw; rr < Cfg::BK; rr += NW) {
                            const int e = lo + j * Cfg::BK + rr;
                            int key = e < hi ? list_s[e] : fallback;
                            if (!IC_DCHECK(key >= 0 && key < p.n_k)) key = 0;
                            const __nv_bfloat16* src = kvb + static_cast<int64_t>(key) * Cfg::DQK;
                            const uint32_t row_dst = tile + (rr >> 3) * 1024 + (rr & 7) * 128;
                            const int x = rr & 7;
#pragma unroll
                            for (int i = 0; i < UPL; ++i) {
                                const int u = lane + 32 * i;
                                if (u < UPR) {
                                    const int u16 = Cfg::TMA_CH * 8 + u;
                                    const uint32_t dst =
                                        row_dst + (u16 >> 3) * Cfg::CH_BYTES + (((u16 & 7) ^ x) << 4);
                                    cp_async_16(dst, src + u16 * 8);
                                }
                            }
                        }
                        cp_async_mbar_arrive_noinc(bar_kv_full(s));
                    }
                    ++kv_n;
                }
                ++q_n;
            }
            // list_s and cnt_s are rewritten by the next row's compaction
            named_bar_sync(3, Cfg::NPROD);
        }
      } else {
        // ------------------------------------------------------------ MMA issuer
        uint32_t kv_n = 0, pv_n = 0, q_n = 0;
        for (int r = 0; r < n_rounds; ++r) {
            const int item = attn_snake(r, blockIdx.x, gridDim.x);
            if (item >= p.n_work) continue;
            const AttnWork wk = attn_work(p, item);
            const int n_valid = warp_count_valid(p.idx + wk.row * p.topk, p.topk, p.n_k, lane);
            const int len = ceil_div(ceil_div(n_valid, p.n_splits), Cfg::BK) * Cfg::BK;
            const int lo = min(n_valid, wk.split * len);
            const int hi = min(n_valid, lo + len);
            const int n_tiles = ceil_div(hi - lo, Cfg::BK);
            if (n_tiles == 0) continue;
            if (lane == 0) {
                mbar_wait(bar_q_full, q_n & 1, abort_flag);
                tc_fence_after();
                // Issue order: QK(j), with PV(j-1) slotted in between QK(j)'s
                // chunks as soon as P(j-1) is ready; PV(j-1) frees tile j-1's
                // stage, whose refill (tile j+1) then overlaps the rest of QK(j).
                auto pv_ready = [&](int j) {
                    const int s = pv_n & 1;
                    return mbar_test_wait(bar_p_full(s), (pv_n >> 1) & 1) &&
                           (j != 1 || mbar_test_wait(bar_o_free, (q_n & 1) ^ 1));
                };
                auto issue_pv = [&](int j) {
                    // O^T += V^T . P^T for tile j-1
                    const int s = pv_n & 1;
                    const bool go = mbar_wait(bar_p_full(s), (pv_n >> 1) & 1, abort_flag) &&
                                    (j != 1 || mbar_wait(bar_o_free, (q_n & 1) ^ 1, abort_flag));
                    tc_fence_after();
                    if (!go) {  // aborted: issue nothing more; the teardown drains
                        ++pv_n;
                        return;
                    }
                    const uint32_t tile = s_base + Cfg::OFF_T + s * Cfg::TILE_BYTES;
                    const uint64_t adesc0 = make_sw128_desc(tile, Cfg::CH_BYTES, 1024);
                    const uint64_t bdesc0 = make_sw128_desc(tile + Cfg::P_CHUNK * Cfg::CH_BYTES, Cfg::CH_BYTES, 1024);
                    const uint32_t first = j > 1 ? 1u : 0u;
#pragma unroll
                    for (int vb = 0; vb < Cfg::NVB; ++vb) {
#pragma unroll
                        for (int ks = 0; ks < Cfg::BK / 16; ++ks) {
                            const uint32_t a_off = ((vb * Cfg::VB_M / 64) * Cfg::CH_BYTES + ks * 2048) >> 4;
                            mma_f16(tmem_base + Cfg::O_COL + 64 * vb, adesc0 + a_off, bdesc0 + ((ks * 2048) >> 4),
                                    Cfg::IDESC_O, (first | ks) ? 1u : 0u);
                        }
                    }
                    mma_commit(bar_kv_empty(s));
                    mma_commit(bar_pv_done);
                    ++pv_n;
                };
                for (int j = 0; j <= n_tiles; ++j) {
                    bool pv_done_here = j == 0;
                    if (j < n_tiles) {
                        // S^T_j = K_j . Q^T into S buffer (tile parity)
                        const int s = kv_n & 1;
                        bool go = mbar_wait(bar_kv_full(s), (kv_n >> 1) & 1, abort_flag);
                        fence_proxy_async_smem();  // cp.async-written chunks before the MMA reads
                        go = mbar_wait(bar_s_free(s), ((kv_n >> 1) & 1) ^ 1, abort_flag) && go;
                        tc_fence_after();
                        if (!go) {  // aborted: issue nothing more; the teardown drains
                            ++kv_n;
                            continue;
                        }
                        // descriptors: base + (byte offset >> 4) in the start-address field
                        const uint64_t adesc0 = make_sw128_desc(s_base + Cfg::OFF_T + s * Cfg::TILE_BYTES);
                        const uint64_t bdesc0 = make_sw128_desc(s_base + Cfg::OFF_Q);
                        const uint32_t d_s = tmem_base + Cfg::S_COL + 64 * s;
#pragma unroll
                        for (int ch = 0; ch < Cfg::NCH; ++ch) {
#pragma unroll
                            for (int k4 = 0; k4 < 4; ++k4) {
                                const int ks = ch * 4 + k4;
                                const uint32_t a_off = (ch * Cfg::CH_BYTES + k4 * 32) >> 4;
                                const uint32_t b_off = (ch * Cfg::Q_CH_BYTES + k4 * 32) >> 4;
                                mma_f16(d_s, adesc0 + a_off, bdesc0 + b_off, Cfg::IDESC_S, ks > 0 ? 1u : 0u);
                            }
                            if (!pv_done_here && ch + 1 < Cfg::NCH && pv_ready(j)) {
                                issue_pv(j);
                                pv_done_here = true;
                            }
                        }
                        mma_commit(bar_s_full(s));
                        if (j == n_tiles - 1) mma_commit(bar_q_empty);
                        ++kv_n;
                    }
                    if (!pv_done_here) issue_pv(j);
                }
            }
            __syncwarp();
            ++q_n;
        }
        }
    } else {
        regs_inc<Cfg::REGS_SOFTMAX>();
        // ------------------------------------------------- softmax and output
        const int wq = warp & 3;               // TMEM lane quarter
        const int sw = warp >> 2;              // softmax warpgroup
        const int hb = Cfg::SMX_HEADS * sw;    // its heads: [hb, hb + 32)
        const int wtid = threadIdx.x - 128 * sw;
        const int sbar = 1 + sw;               // its named barrier
        uint32_t t_it = 0;  // tiles (and so P.V products) handled so far
        for (int r = 0; r < n_rounds; ++r) {
            const int item = attn_snake(r, blockIdx.x, gridDim.x);
            if (item >= p.n_work) continue;
            const AttnWork wk = attn_work(p, item);
            const int n_valid = warp_count_valid(p.idx + wk.row * p.topk, p.topk, p.n_k, lane);
            const int len = ceil_div(ceil_div(n_valid, p.n_splits), Cfg::BK) * Cfg::BK;
            const int lo = min(n_valid, wk.split * len);
            const int hi = min(n_valid, lo + len);
            const int n_tiles = ceil_div(hi - lo, Cfg::BK);

            // Each thread owns a quarter of one key's heads: key (within the
            // warp's 16) = 8*(lane&1) + (lane>>2), heads hb + 2r + par, r < 16.
            const int par = (lane >> 1) & 1;
            const int key_in_tile = wq * 16 + 8 * (lane & 1) + (lane >> 2);
            float l_part[16];
#pragma unroll
            for (int r2 = 0; r2 < 16; ++r2) l_part[r2] = 0.f;

            for (int j = 0; j < n_tiles; ++j) {
                const int st = t_it & 1;
                mbar_wait(bar_s_full(st), (t_it >> 1) & 1, abort_flag);
                tc_fence_after();
                uint32_t sv[16];
                tmem_ld_16x64b_x16(tmem_base + (static_cast<uint32_t>(wq * 32) << 16) + Cfg::S_COL + 64 * st + hb,
                                   sv);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_s_free(st));
                const bool valid = (lo + j * Cfg::BK + key_in_tile) < hi;
                if (j == 0) {
                    // reference logit per head: the first key of this slice
                    if (wq == 0 && (lane & ~2) == 0) {
#pragma unroll
                        for (int r2 = 0; r2 < 16; ++r2)
                            m_s[hb + 2 * r2 + par] = __fmul_rn(__uint_as_float(sv[r2]), p.sm_scale_log2);
                    }
                    named_bar_sync(sbar, 128);
                }
                // z = logit (log2 units) minus the per-head reference, in place
                float zmax = -INFINITY;
#pragma unroll
                for (int r2 = 0; r2 < 16; ++r2) {
                    const float z = __fmul_rn(__uint_as_float(sv[r2]), p.sm_scale_log2) - m_s[hb + 2 * r2 + par];
                    zmax = fmaxf(zmax, valid ? z : -INFINITY);
                    sv[r2] = __float_as_uint(z);
                }
                if (named_bar_or(sbar, 128, zmax > IC_ATTN_RESCALE_LOG2)) {
                    // rare path: raise the reference to the tile maximum and
                    // rescale the accumulated output and row sums
                    float tmax[16];
#pragma unroll
                    for (int r2 = 0; r2 < 16; ++r2) tmax[r2] = valid ? __uint_as_float(sv[r2]) : -INFINITY;
#pragma unroll
                    for (int r2 = 0; r2 < 16; ++r2) {
                        tmax[r2] = fmaxf(tmax[r2], __shfl_xor_sync(0xffffffffu, tmax[r2], 1));
                        tmax[r2] = fmaxf(tmax[r2], __shfl_xor_sync(0xffffffffu, tmax[r2], 4));
                        tmax[r2] = fmaxf(tmax[r2], __shfl_xor_sync(0xffffffffu, tmax[r2], 8));
                        tmax[r2] = fmaxf(tmax[r2], __shfl_xor_sync(0xffffffffu, tmax[r2], 16));
                    }
                    if ((lane & ~2) == 0) {
#pragma unroll
                        for (int r2 = 0; r2 < 16; ++r2) red_s[wq * 64 + hb + 2 * r2 + par] = tmax[r2];
                    }
                    named_bar_sync(sbar, 128);
                    if (wtid < Cfg::SMX_HEADS) {
                        // red_s holds max(z) relative to the old reference
                        const int h = hb + wtid;
                        float dz = 0.f;
                        for (int w4 = 0; w4 < 4; ++w4) dz = fmaxf(dz, red_s[w4 * 64 + h]);
                        a_s[h] = dz;  // reference shift; earlier terms scale by 2^-dz
                        m_s[h] += dz;
                    }
                    named_bar_sync(sbar, 128);
#pragma unroll
                    for (int r2 = 0; r2 < 16; ++r2) {
                        const float dz = a_s[hb + 2 * r2 + par];
                        l_part[r2] *= ex2_approx(-dz);
                        sv[r2] = __float_as_uint(__uint_as_float(sv[r2]) - dz);
                    }
                    if (j >= 1) {
                        // the previous tile's P.V must be complete before the
                        // accumulator is rescaled. P.V(j-2) was issued before
                        // QK(j) and the MMAs complete in issue order, so with S(j)
                        // in hand the barrier is at most one phase behind P.V(j-1):
                        // the parity wait is exact (P.V count = tile count)
                        mbar_wait(bar_pv_done, (t_it - 1) & 1, abort_flag);
                        tc_fence_after();
                        for (int vb = 0; vb < Cfg::NVB; ++vb) {
                            {
                                const int half = sw;
                                uint32_t o32[32];
                                const uint32_t ta = tmem_base + (static_cast<uint32_t>(wq * 32) << 16) +
                                                    Cfg::O_COL + 64 * vb + 32 * half;
                                tmem_ld<32>(ta, o32);
                                tmem_wait_ld();
#pragma unroll
                                for (int c = 0; c < 32; ++c)
                                    o32[c] = __float_as_uint(__uint_as_float(o32[c]) *
                                                             ex2_approx(-a_s[32 * half + c]));
                                tmem_st32(ta, o32);
                            }
                        }
                        tmem_wait_st();
                    }
                    named_bar_sync(sbar, 128);
                }
                // probabilities and row sums
#pragma unroll
                for (int r2 = 0; r2 < 16; ++r2) {
                    const float pr = valid ? ex2_approx(__uint_as_float(sv[r2])) : 0.f;
                    l_part[r2] += pr;
                    sv[r2] = __float_as_uint(pr);
                }
                // bf16 P^T row of this key: this thread writes heads
                // [hb + 16 par, hb + 16 par + 16), pairing its own column with its
                // partner's (lane ^ 2)
                uint32_t packed[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float send = par ? __uint_as_float(sv[i]) : __uint_as_float(sv[8 + i]);
                    const float mine = par ? __uint_as_float(sv[8 + i]) : __uint_as_float(sv[i]);
                    const float other = __shfl_xor_sync(0xffffffffu, send, 2);
                    packed[i] = par ? pack_bf16x2(other, mine) : pack_bf16x2(mine, other);
                }
                const uint32_t prow = s_base + Cfg::OFF_T + st * Cfg::TILE_BYTES +
                                      Cfg::P_CHUNK * Cfg::CH_BYTES + (key_in_tile >> 3) * 1024 +
                                      (key_in_tile & 7) * 128;
#pragma unroll
                for (int u2 = 0; u2 < 2; ++u2) {
                    const int u = hb / 8 + 2 * par + u2;
                    st_shared_v4(prow + ((u ^ (key_in_tile & 7)) << 4), packed[4 * u2], packed[4 * u2 + 1],
                                 packed[4 * u2 + 2], packed[4 * u2 + 3]);
                }
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_p_full(st));
                ++t_it;
            }

            // ---- end of row: row sums, then the output (or the partials), once
            // the row's last two P.V are complete (P.V(n-3) was issued before
            // QK(n-1), so the barrier is at most two phases behind: wait for
            // the second-to-last, then the last, each an exact parity wait)
            if (n_tiles > 0) {
                if (n_tiles >= 2) mbar_wait(bar_pv_done, (t_it - 2) & 1, abort_flag);
                mbar_wait(bar_pv_done, (t_it - 1) & 1, abort_flag);
                tc_fence_after();
            }
#pragma unroll
            for (int r2 = 0; r2 < 16; ++r2) {
                l_part[r2] += __shfl_xor_sync(0xffffffffu, l_part[r2], 1);
                l_part[r2] += __shfl_xor_sync(0xffffffffu, l_part[r2], 4);
                l_part[r2] += __shfl_xor_sync(0xffffffffu, l_part[r2], 8);
                l_part[r2] += __shfl_xor_sync(0xffffffffu, l_part[r2], 16);
            }
            if ((lane & ~2) == 0) {
#pragma unroll
                for (int r2 = 0; r2 < 16; ++r2) red_s[wq * 64 + hb + 2 * r2 + par] = l_part[r2];
            }
            named_bar_sync(sbar, 128);
            if (wtid < Cfg::SMX_HEADS) {
                const int h = hb + wtid;
                const float l = red_s[h] + red_s[64 + h] + red_s[128 + h] + red_s[192 + h];
                if (p.n_splits == 1) {
                    a_s[h] = l > 0.f ? 1.0f / l : 0.f;
                } else {
                    a_s[h] = l;
                }
            }
            named_bar_sync(sbar, 128);
            const int64_t slot = wk.row * p.n_splits + wk.split;
            if (p.n_splits > 1 && wtid < Cfg::SMX_HEADS) {
                const int h = hb + wtid;
                p.ml_part[slot * 128 + h] = n_tiles > 0 ? m_s[h] : -INFINITY;
                p.ml_part[slot * 128 + 64 + h] = n_tiles > 0 ? a_s[h] : 0.f;
            }
            for (int vb = 0; vb < Cfg::NVB; ++vb) {
                const bool row_ok = Cfg::VB_M == 128 || lane < 16;
                const int v = vb * Cfg::VB_M + (Cfg::VB_M == 128 ? wq * 32 + lane : wq * 16 + lane);
                {
                    const int half = sw;
                    uint32_t o32[32];
                    if (n_tiles > 0) {
                        tmem_ld<32>(tmem_base + (static_cast<uint32_t>(wq * 32) << 16) + Cfg::O_COL +
                                        64 * vb + 32 * half,
                                    o32);
                        tmem_wait_ld();
                    } else {
#pragma unroll
                        for (int c = 0; c < 32; ++c) o32[c] = 0u;
                    }
                    if (row_ok) {
#pragma unroll
                        for (int c = 0; c < 32; ++c) {
                            const int h = 32 * half + c;
                            if (h < p.H) {
                                const float o = __uint_as_float(o32[c]);
                                if (p.n_splits == 1) {
                                    p.out[(wk.row * p.H + h) * Cfg::DV + v] = __float2bfloat16_rn(o * a_s[h]);
                                } else {
                                    p.o_part[(slot * p.H + h) * Cfg::DV + v] = o;
                                }
                            }
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (n_tiles > 0 && lane == 0) mbar_arrive(bar_o_free);
            named_bar_sync(sbar, 128);
        }
    }

    __syncthreads();
    if (*abort_flag) {  // final after the barrier: the same in every thread
        // let the copies and MMAs issued before the abort land before the
        // shared and tensor memory they write goes away
        if (warp >= 8 && warp != MMA_WARP) {
            cp_async_wait_all();
            if (warp == 8 && lane == 0) {
                if (q_armed > 0) mbar_drain(bar_q_full, (q_armed - 1) & 1);
                // a tile's phase also needs every producer thread's cp.async
                // arrival, so after an abort it may never complete: the drain
                // then gives up after its bound
                for (uint32_t i = kv_armed > 2 ? kv_armed - 2 : 0; i < kv_armed; ++i)
                    mbar_drain(bar_kv_full(i & 1), (i >> 1) & 1);
            }
        }
        if (warp == MMA_WARP && lane == 0) {
            mma_commit(bar_drain);
            mbar_drain(bar_drain, 0);
        }
        __syncthreads();
    }
    if (warp == MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
    }
}

// Merge split partials: out[h,v] = sum_c 2^(m_c - M) O_c[h,v] / sum_c 2^(m_c - M) l_c.
template <int DV>
__global__ void __launch_bounds__(128)
    attn_combine_kernel(const float* __restrict__ o_part, const float* __restrict__ ml_part,
                        int n_splits, int H, __nv_bfloat16* __restrict__ out) {
    // one CTA per (row, head); every thread derives the split weights itself
    // from the per-split running maximum m (log2 units) and sum l
    griddep_sync();  // the partials come from the previous kernel
    const int64_t row = blockIdx.x / H;
    const int h = blockIdx.x % H;
    float m_c[8], w_c[8];
    float M = -INFINITY;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        m_c[c] = c < n_splits ? __ldg(ml_part + (row * n_splits + c) * 128 + h) : -INFINITY;
        M = fmaxf(M, m_c[c]);
    }
    float lsum = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        w_c[c] = (m_c[c] == -INFINITY) ? 0.f : ex2_approx(m_c[c] - M);
        if (c < n_splits) lsum += w_c[c] * __ldg(ml_part + (row * n_splits + c) * 128 + 64 + h);
    }
    const float inv_l = lsum > 0.f ? 1.0f / lsum : 0.f;
    for (int i = 4 * threadIdx.x; i < DV; i += 4 * blockDim.x) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            if (c < n_splits) {
                const float4 v = __ldg(reinterpret_cast<const float4*>(
                    o_part + ((row * n_splits + c) * H + h) * DV + i));
                acc.x += w_c[c] * v.x;
                acc.y += w_c[c] * v.y;
                acc.z += w_c[c] * v.z;
                acc.w += w_c[c] * v.w;
            }
        }
        __nv_bfloat16* dst = out + (row * H + h) * DV + i;
        const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x * inv_l, acc.y * inv_l);
        const __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z * inv_l, acc.w * inv_l);
        if ((reinterpret_cast<uintptr_t>(dst) & 7u) == 0) {
            uint2 pk;
            pk.x = *reinterpret_cast<const uint32_t*>(&lo);
            pk.y = *reinterpret_cast<const uint32_t*>(&hi);
            *reinterpret_cast<uint2*>(dst) = pk;
        } else {
            dst[0] = lo.x;
            dst[1] = lo.y;
            dst[2] = hi.x;
            dst[3] = hi.y;
        }
    }
}

}  // namespace ic
