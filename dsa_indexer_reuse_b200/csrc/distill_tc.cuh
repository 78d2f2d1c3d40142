// Multi-layer distillation target on the tensor cores (sm_100a), for the
// model's shapes: 64 attention heads over d_qk-wide latent rows, and a
// 64-head, 128-wide indexer (bf16, or FP8 E4M3 with per-token scales).
//
// It computes what distill_target_kernel computes (IndexCache paper, Abstract:
// each retained indexer is trained against the averaged attention
// distributions of the layers it serves; Table 3, "w/o cross-layer loss"): for
// query row r and the valid keys s_j of the Full layer's index row,
//   P[j]  = (1 / (n_served * H)) sum_l sum_h softmax_j(sm_scale * q_l[r,h,:] . kv_l[s_j,:])
//   Q[j]  = softmax_j(I[r, s_j]),   kl[r] = sum_j P[j] (log P[j] - log Q[j]).
//
// Mapping (one query row per CTA iteration, persistent CTAs):
//  * The valid keys of the row are compacted in order (key slot = rank among
//    the row's valid entries) and taken 128 at a time: a tile is one MMA M.
//  * The logits of a tile are S^T = K_tile . Q^T on tcgen05 (M = 128 keys,
//    N = 64 heads, K = d_qk, bf16 in, fp32 out), so TMEM lane i holds key i's
//    64 head logits. The tile's rows are gathered from global memory in
//    128-byte column chunks (16 KB per chunk) through a ring of shared-memory
//    slots; the query rows stay resident, 128-byte swizzled, K-major.
//  * Tensor memory holds eight 64-column accumulators. A head's softmax needs
//    its normaliser over all keys before any probability is final, so every
//    tile's logits are read twice: a statistics pass (a running max and sum of
//    exponentials per head and per thread, merged across the keys' threads at
//    the end) and a probability pass. The last eight tiles of a row-layer stay
//    in tensor memory between the two passes; the logits of earlier tiles (up
//    to 8 x 32 KB per CTA) wait in a global workspace, which costs less than
//    gathering and multiplying those tiles again.
//  * The indexer scores of the same keys use the same machinery (K = 128:
//    kind::f16 for bf16, kind::f8f6f4 for E4M3), followed by ReLU, the head
//    weights and the scales in the epilogue; then the softmax of the scores
//    and the KL as block reductions, and the target row is written back at
//    the index row's positions (0 at invalid ones).
//
// Warp roles (512 threads): warps 0-3 epilogue (one thread per TMEM lane),
// warp 4 MMA issuer and TMEM owner, warps 5-12 the cp.async gathers of
// key-row chunks, warps 13-15 the index compaction, the query-row loads and
// L2 prefetches of the row's selected keys, one row ahead of the gathers.
#pragma once

#include "distill.cuh"

namespace ic {

template <int DQK_, bool FP8I_>
struct DistTcCfg {
    static constexpr int DQK = DQK_;
    static constexpr bool FP8I = FP8I_;
    static_assert(DQK % 64 == 0 && DQK <= 576, "d_qk");
    static constexpr int H = 64;                   // attention heads (MMA N)
    static constexpr int HI = 64;                  // indexer heads (MMA N)
    static constexpr int DI = 128;                 // indexer head width
    static constexpr int BM = 128;                 // keys per tile (MMA M, TMEM lanes)
    static constexpr int NCH = DQK / 64;           // 128-byte chunks of a latent row
    static constexpr int NCH_I = FP8I ? 1 : 2;     // 128-byte chunks of an indexer key row
    static constexpr int CH_BYTES = BM * 128;      // one ring slot: 128 rows x 128 B
    static constexpr int NS = 6;                   // ring slots
    static constexpr int NSLOT = 8;                // TMEM accumulators of 64 columns
    static constexpr int RESIDENT = NSLOT;         // tiles kept between the two passes
    // logits of the other tiles of a row-layer (at most MAX_TOPK / BM - RESIDENT),
    // fp32, per CTA: [tile][16 groups of 4 heads][128 keys] float4
    static constexpr int SPILL_TILES = 2048 / BM - RESIDENT;
    static constexpr size_t SPILL_BYTES_PER_CTA = static_cast<size_t>(SPILL_TILES) * BM * 64 * 4;
    static constexpr int MAX_TOPK = 2048;
    static constexpr int THREADS = 512;
    static constexpr int MMA_WARP = 4;
    static constexpr int AUX_WARP0 = 13;           // warps 5..12 gather key rows, 13..15 the rest
    static constexpr int NGATHER = 32 * (AUX_WARP0 - MMA_WARP - 1);
    static constexpr int NAUX = 32 * (16 - AUX_WARP0);
    static_assert(NGATHER == 256, "four 16-byte units of every 128-row chunk per gather thread");
    static constexpr int REGS_EPI = 200, REGS_OTHER = 104;
    static_assert(128 * REGS_EPI + 384 * REGS_OTHER <= 65536, "register split");
    static constexpr uint32_t IDESC_S = make_idesc(BM, H, FMT_BF16, FMT_BF16);
    static constexpr uint32_t IDESC_I =
        make_idesc(BM, HI, FP8I ? FMT_E4M3 : FMT_BF16, FP8I ? FMT_E4M3 : FMT_BF16);
    static constexpr int Q_CH_BYTES = H * 128;     // one 128-byte column chunk of 64 rows
    // shared memory layout (byte offsets)
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_QI = OFF_Q + NCH * Q_CH_BYTES;
    static constexpr int OFF_RING = OFF_QI + NCH_I * Q_CH_BYTES;
    static constexpr int OFF_LIST = OFF_RING + NS * CH_BYTES;      // [2][MAX_TOPK] keys
    static constexpr int OFF_P = OFF_LIST + 2 * MAX_TOPK * 4;      // [MAX_TOPK] target
    static constexpr int OFF_Z = OFF_P + MAX_TOPK * 4;             // [MAX_TOPK] indexer scores
    static constexpr int OFF_HM = OFF_Z + MAX_TOPK * 4;            // [64] head max (log2 units)
    static constexpr int OFF_HL = OFF_HM + 64 * 4;                 // [64] 1 / head sum
    static constexpr int OFF_RED = OFF_HL + 64 * 4;                // [4][64][2] warp partials
    static constexpr int OFF_W = OFF_RED + 4 * 64 * 2 * 4;         // [64] w * q_scale
    static constexpr int OFF_MISC = OFF_W + 64 * 4;                // counts, scan scratch
    static constexpr int OFF_BAR = OFF_MISC + 128;
    // mbarriers: ring_full[NS], ring_empty[NS], acc_full[NSLOT], acc_empty[NSLOT],
    // q_full, q_empty, qi_full, qi_empty, list_full[2], list_free[2], drain
    static constexpr int NUM_BARS = 2 * NS + 2 * NSLOT + 9;
    static constexpr int OFF_TSLOT = OFF_BAR + NUM_BARS * 8;       // TMEM base, abort flag
    static constexpr int SMEM_BYTES = OFF_TSLOT + 16;
    static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;           // slack for 1024-byte alignment
    static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
};

// Number of tiles of a row of n valid keys.
__device__ __forceinline__ int dist_tiles(int n) { return (n + 127) >> 7; }

// Tiles of a row-layer that do not stay in tensor memory between the two
// passes: the first T - RESIDENT, whose logits wait in the spill workspace.
template <class Cfg>
__device__ __forceinline__ int dist_spilled(int T) {
    return T > Cfg::RESIDENT ? T - Cfg::RESIDENT : 0;
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, 1) distill_tc_kernel(const __grid_constant__ DistillParams p) {
    constexpr int NS = Cfg::NS, NSLOT = Cfg::NSLOT, NCH = Cfg::NCH, NCH_I = Cfg::NCH_I;
    constexpr int MMA_WARP = Cfg::MMA_WARP, DQK = Cfg::DQK;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align_smem_1024(smem_raw);
    const uint32_t s_base = smem_u32(smem);
    int32_t* list_s = reinterpret_cast<int32_t*>(smem + Cfg::OFF_LIST);
    float* P_s = reinterpret_cast<float*>(smem + Cfg::OFF_P);
    float* Z_s = reinterpret_cast<float*>(smem + Cfg::OFF_Z);
    float* hm_s = reinterpret_cast<float*>(smem + Cfg::OFF_HM);
    float* hl_s = reinterpret_cast<float*>(smem + Cfg::OFF_HL);
    float* red_s = reinterpret_cast<float*>(smem + Cfg::OFF_RED);
    float* w_s = reinterpret_cast<float*>(smem + Cfg::OFF_W);
    int* misc_s = reinterpret_cast<int*>(smem + Cfg::OFF_MISC);  // [0,2): n per list buffer; [8,11), [24,28): scans
    const uint32_t bar0 = s_base + Cfg::OFF_BAR;
    auto bar_ring_full = [&](int s) { return bar0 + 8u * s; };
    auto bar_ring_empty = [&](int s) { return bar0 + 8u * (NS + s); };
    auto bar_acc_full = [&](int s) { return bar0 + 8u * (2 * NS + s); };
    auto bar_acc_empty = [&](int s) { return bar0 + 8u * (2 * NS + NSLOT + s); };
    const uint32_t bar_q_full = bar0 + 8u * (2 * NS + 2 * NSLOT);
    const uint32_t bar_q_empty = bar_q_full + 8u, bar_qi_full = bar_q_full + 16u, bar_qi_empty = bar_q_full + 24u;
    auto bar_list_full = [&](int b) { return bar_q_full + 32u + 8u * b; };
    auto bar_list_free = [&](int b) { return bar_q_full + 48u + 8u * b; };
    const uint32_t bar_drain = bar_q_full + 64u;
    static_assert(Cfg::NUM_BARS == 2 * NS + 2 * NSLOT + 9, "barrier slots");
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Cfg::OFF_TSLOT);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Cfg::OFF_TSLOT + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(bar_ring_full(s), Cfg::NGATHER);
            mbar_init(bar_ring_empty(s), 1);
        }
        for (int s = 0; s < NSLOT; ++s) {
            mbar_init(bar_acc_full(s), 1);
            mbar_init(bar_acc_empty(s), 4);
        }
        mbar_init(bar_q_full, Cfg::NAUX);
        mbar_init(bar_q_empty, 1);
        mbar_init(bar_qi_full, Cfg::NAUX);
        mbar_init(bar_qi_empty, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(bar_list_full(b), 1);
            mbar_init(bar_list_free(b), 1);
        }
        mbar_init(bar_drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == MMA_WARP) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int rows = p.rows;
    const int n_rounds = ceil_div(rows, static_cast<int>(gridDim.x));
    auto row_of = [&](int r) { return rows - 1 - (r * static_cast<int>(gridDim.x) + static_cast<int>(blockIdx.x)); };
    const int L = p.n_served;

    if (warp >= 4) {
      regs_dec<Cfg::REGS_OTHER>();
      if (warp != MMA_WARP) {
        if (warp < Cfg::AUX_WARP0) {
        // --------------------------------------------- key-row chunk gathers
        // Thread gt copies 16-byte unit x = gt % 8 of rows gt / 8 + 32 k
        // (k = 0..3) of every chunk: the same four rows for all chunks of a
        // tile, so a tile's source rows are looked up once.
        const int gt = threadIdx.x - 32 * (Cfg::MMA_WARP + 1);  // 0 .. NGATHER-1
        const int x = gt & 7, r8 = (gt >> 3) & 7;
        uint32_t dst_off[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) dst_off[k] = ((gt >> 6) + 4 * k) * 1024 + r8 * 128 + ((x ^ r8) << 4);
        uint32_t ring_n = 0;  // chunks filled so far
        for (int r = 0; r < n_rounds; ++r) {
            const int row = row_of(r);
            if (row < 0) continue;
            const int buf = r & 1;
            mbar_wait(bar_list_full(buf), (r >> 1) & 1, abort_flag);
            const int n = misc_s[buf];
            if (n == 0) continue;
            const int32_t* lst = list_s + buf * Cfg::MAX_TOPK;
            const int T = dist_tiles(n);
            const int b = row / p.n_q;
            // the `nch` 128-byte chunks of the keys of `tile`, one ring slot each
            auto gather_tile = [&](const uint8_t* base, int row_bytes, int nch, int tile) {
                const uint8_t* src[4];
                uint32_t bytes[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int slot = tile * Cfg::BM + (gt >> 3) + 32 * k;
                    const int key = slot < n ? lst[slot] : -1;
                    src[k] = base + static_cast<int64_t>(key < 0 ? 0 : key) * row_bytes + x * 16;
                    bytes[k] = key < 0 ? 0u : 16u;
                }
                for (int c = 0; c < nch; ++c) {
                    const int s = static_cast<int>(ring_n % NS);
                    if (mbar_wait(bar_ring_empty(s), ((ring_n / NS) & 1) ^ 1, abort_flag)) {
                        const uint32_t dst0 = s_base + Cfg::OFF_RING + s * Cfg::CH_BYTES;
#pragma unroll
                        for (int k = 0; k < 4; ++k) cp_async_16_zfill(dst0 + dst_off[k], src[k] + c * 128, bytes[k]);
                        cp_async_mbar_arrive_noinc(bar_ring_full(s));
                    }
                    ++ring_n;
                }
            };
            for (int l = 0; l < L; ++l) {
                const uint8_t* kvb = reinterpret_cast<const uint8_t*>(p.kv[l] + static_cast<int64_t>(b) * p.n_k * DQK);
                for (int t = 0; t < T; ++t) gather_tile(kvb, DQK * 2, NCH, t);
            }
            const int ibytes = Cfg::DI * (Cfg::FP8I ? 1 : 2);
            const uint8_t* kib = reinterpret_cast<const uint8_t*>(p.k_I) + static_cast<int64_t>(b) * p.n_k * ibytes;
            for (int t = 0; t < T; ++t) gather_tile(kib, ibytes, NCH_I, t);
        }
        cp_async_wait_all();
        } else {
        // ------------------- index compaction, query rows and L2 prefetches
        const int at = threadIdx.x - 32 * Cfg::AUX_WARP0;  // 0 .. NAUX-1
        const int aw = at >> 5;
        constexpr int NAUX = Cfg::NAUX;
        int q_n = 0, qi_n = 0;
        // 64 rows of `row_bytes` (a query's heads) into 128-byte swizzled chunks at dst0
        auto load_rows64 = [&](uint32_t dst0, const uint8_t* src0, int row_bytes, uint32_t bar) {
            const int upr = row_bytes / 16;  // 16-byte units per row
            for (int u = at; u < 64 * upr; u += NAUX) {
                const int h = u / upr, c16 = u % upr;
                const int ch = c16 >> 3, xx = c16 & 7;
                const uint32_t dst = dst0 + ch * Cfg::Q_CH_BYTES + (h >> 3) * 1024 + (h & 7) * 128 + ((xx ^ (h & 7)) << 4);
                cp_async_16(dst, src0 + static_cast<int64_t>(h) * row_bytes + c16 * 16);
            }
            cp_async_mbar_arrive_noinc(bar);
        };
        for (int r = 0; r < n_rounds; ++r) {
            const int row = row_of(r);
            if (row < 0) continue;
            const int buf = r & 1;
            int32_t* lst = list_s + buf * Cfg::MAX_TOPK;
            // the buffer's previous row (two rows back) must be finished
            mbar_wait(bar_list_free(buf), ((r >> 1) & 1) ^ 1, abort_flag);
            // ordered compaction of the valid entries of the index row
            const int32_t* irow = p.idx + static_cast<int64_t>(row) * p.topk;
            int run = 0;
            for (int e0 = 0; e0 < p.topk; e0 += NAUX) {
                const int e = e0 + at;
                const int s = e < p.topk ? irow[e] : -1;
                const bool ok = s >= 0 && s < p.n_k;
                const uint32_t bal = __ballot_sync(0xffffffffu, ok);
                if (lane == 0) misc_s[8 + aw] = __popc(bal);
                named_bar_sync(2, NAUX);
                int before = 0, total = 0;
#pragma unroll
                for (int w = 0; w < NAUX / 32; ++w) {
                    const int c = misc_s[8 + w];
                    before += w < aw ? c : 0;
                    total += c;
                }
                if (ok) {
                    const int slot = run + before + __popc(bal & lanemask_lt());
                    if (IC_DCHECK(slot < Cfg::MAX_TOPK)) lst[slot] = s;
                }
                run += total;
                named_bar_sync(2, NAUX);  // misc_s is rewritten by the next chunk
            }
            const int n = run;
            if (at == 0) {
                misc_s[buf] = n;
                mbar_arrive(bar_list_full(buf));  // release: the list and its count
            }
            if (n == 0) continue;
            const int b = row / p.n_q;
            // every layer's query rows and selected key rows are requested from L2
            // ahead of their loads
            {
                const int ib = Cfg::DI * (Cfg::FP8I ? 1 : 2);
                for (int u = at; u <= L; u += NAUX) {
                    if (u < L)
                        prefetch_l2_bulk(p.q[u] + static_cast<int64_t>(row) * Cfg::H * DQK, Cfg::H * DQK * 2);
                    else
                        prefetch_l2_bulk(reinterpret_cast<const uint8_t*>(p.q_I) + static_cast<int64_t>(row) * Cfg::HI * ib,
                                         Cfg::HI * ib);
                }
            }
            for (int l = 0; l < L; ++l) {
                const uint8_t* kvb = reinterpret_cast<const uint8_t*>(p.kv[l] + static_cast<int64_t>(b) * p.n_k * DQK);
                for (int j = at; j < n; j += NAUX) prefetch_l2_bulk(kvb + static_cast<int64_t>(lst[j]) * DQK * 2, DQK * 2);
            }
            for (int l = 0; l < L; ++l) {
                if (mbar_wait(bar_q_empty, (q_n & 1) ^ 1, abort_flag))
                    load_rows64(s_base + Cfg::OFF_Q,
                                reinterpret_cast<const uint8_t*>(p.q[l] + static_cast<int64_t>(row) * Cfg::H * DQK), DQK * 2,
                                bar_q_full);
                ++q_n;
            }
            const int ibytes = Cfg::DI * (Cfg::FP8I ? 1 : 2);
            if (mbar_wait(bar_qi_empty, (qi_n & 1) ^ 1, abort_flag))
                load_rows64(s_base + Cfg::OFF_QI,
                            reinterpret_cast<const uint8_t*>(p.q_I) + static_cast<int64_t>(row) * Cfg::HI * ibytes, ibytes,
                            bar_qi_full);
            ++qi_n;
        }
        cp_async_wait_all();
        }
      } else if (lane == 0) {
        // ------------------------------------------------------ MMA issuer
        uint32_t ring_n = 0, job = 0;
        int q_n = 0, qi_n = 0;
        // one accumulator: `nch` ring chunks of 128 bytes of K against the
        // resident operand at b_base (chunk stride Q_CH_BYTES)
        auto run_job = [&](int nch, uint32_t b_base, uint32_t idesc, bool fp8) {
            const int as = static_cast<int>(job % NSLOT);
            bool go = mbar_wait(bar_acc_empty(as), ((job / NSLOT) & 1) ^ 1, abort_flag);
            const uint32_t d_tmem = tmem_base + as * 64;
            for (int c = 0; c < nch; ++c) {
                const int s = static_cast<int>(ring_n % NS);
                go = mbar_wait(bar_ring_full(s), (ring_n / NS) & 1, abort_flag) && go;
                tc_fence_after();
                if (go) {
                    const uint64_t adesc = make_sw128_desc(s_base + Cfg::OFF_RING + s * Cfg::CH_BYTES);
                    const uint64_t bdesc = make_sw128_desc(b_base + c * Cfg::Q_CH_BYTES);
#pragma unroll
                    for (int k = 0; k < 4; ++k) {  // 32 bytes of K per instruction
                        const uint32_t acc = (c > 0 || k > 0) ? 1u : 0u;
                        if (fp8)
                            mma_f8(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, acc);
                        else
                            mma_f16(d_tmem, adesc + 2 * k, bdesc + 2 * k, idesc, acc);
                    }
                    mma_commit(bar_ring_empty(s));
                }
                ++ring_n;
            }
            if (go) mma_commit(bar_acc_full(as));
            ++job;
        };
        for (int r = 0; r < n_rounds; ++r) {
            const int row = row_of(r);
            if (row < 0) continue;
            const int buf = r & 1;
            mbar_wait(bar_list_full(buf), (r >> 1) & 1, abort_flag);
            const int n = misc_s[buf];
            if (n == 0) continue;
            const int T = dist_tiles(n);
            for (int l = 0; l < L; ++l) {
                mbar_wait(bar_q_full, q_n & 1, abort_flag);
                tc_fence_after();
                ++q_n;
                for (int t = 0; t < T; ++t) run_job(NCH, s_base + Cfg::OFF_Q, Cfg::IDESC_S, false);
                mma_commit(bar_q_empty);  // the query rows may be replaced
            }
            mbar_wait(bar_qi_full, qi_n & 1, abort_flag);
            tc_fence_after();
            ++qi_n;
            for (int t = 0; t < T; ++t) run_job(NCH_I, s_base + Cfg::OFF_QI, Cfg::IDESC_I, Cfg::FP8I);
            mma_commit(bar_qi_empty);
        }
      }
    } else {
        regs_inc<Cfg::REGS_EPI>();
        // ------------------------------------------------------------ epilogue
        const int tid = threadIdx.x;  // = TMEM lane = key within a tile
        const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
        const float c_log2 = p.sm_scale * 1.4426950408889634f;
        const float inv_norm = 1.f / (static_cast<float>(Cfg::H) * static_cast<float>(L));
        float4* spill = reinterpret_cast<float4*>(static_cast<uint8_t*>(p.spill) + Cfg::SPILL_BYTES_PER_CTA * blockIdx.x);
        uint32_t job = 0;
        auto acquire = [&](uint32_t j) {
            mbar_wait(bar_acc_full(static_cast<int>(j % NSLOT)), (j / NSLOT) & 1, abort_flag);
            tc_fence_after();
            return tmem_base + lane_base + static_cast<uint32_t>(j % NSLOT) * 64;
        };
        auto release = [&](uint32_t j) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_acc_empty(static_cast<int>(j % NSLOT)));
        };
        for (int r = 0; r < n_rounds; ++r) {
            const int row = row_of(r);
            if (row < 0) continue;
            const int buf = r & 1;
            mbar_wait(bar_list_full(buf), (r >> 1) & 1, abort_flag);
            const int n = misc_s[buf];
            const int T = dist_tiles(n);
            const int b = row / p.n_q;
            for (int i = tid; i < T * Cfg::BM; i += 128) P_s[i] = 0.f;
            if (tid < Cfg::HI) {
                const int64_t e = static_cast<int64_t>(row) * Cfg::HI + tid;
                const float wv = p.w_is_f32 ? reinterpret_cast<const float*>(p.w)[e]
                                            : __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p.w)[e]);
                w_s[tid] = wv * (p.q_scale ? p.q_scale[row] : 1.f);
            }
            named_bar_sync(1, 128);
            if (n > 0) {
                for (int l = 0; l < L; ++l) {
                    // ---- statistics pass: running (max, sum of 2^(z - max)) per head
                    float m[64], ls[64];
#pragma unroll
                    for (int h = 0; h < 64; ++h) {
                        m[h] = -INFINITY;
                        ls[h] = 0.f;
                    }
                    const uint32_t job0 = job;
                    const int R = dist_spilled<Cfg>(T);
                    for (int t = 0; t < T; ++t) {
                        const uint32_t ta = acquire(job0 + t);
                        const bool valid = t * Cfg::BM + tid < n;
                        float4* sp = spill + static_cast<size_t>(t) * 16 * Cfg::BM + tid;
#pragma unroll
                        for (int half = 0; half < 2; ++half) {
                            uint32_t v[32];
                            tmem_ld<32>(ta + half * 32, v);
                            tmem_wait_ld();
                            if (t < R) {  // this tile's logits wait in the workspace
#pragma unroll
                                for (int g = 0; g < 8; ++g)
                                    sp[(half * 8 + g) * Cfg::BM] =
                                        make_float4(__uint_as_float(v[4 * g]), __uint_as_float(v[4 * g + 1]),
                                                    __uint_as_float(v[4 * g + 2]), __uint_as_float(v[4 * g + 3]));
                            }
                            if (valid) {
#pragma unroll
                                for (int k = 0; k < 32; ++k) {
                                    const int h = half * 32 + k;
                                    const float z = __uint_as_float(v[k]) * c_log2;
                                    const float d = z - m[h];
                                    const float e = ex2_approx(-fabsf(d));
                                    const bool up = d > 0.f;
                                    ls[h] = up ? fmaf(ls[h], e, 1.f) : ls[h] + e;
                                    m[h] = up ? z : m[h];
                                }
                            }
                        }
                        if (t < R) release(job0 + t);
                    }
                    // merge across the warp (a butterfly that halves the heads
                    // held per lane at each step: lane L ends with heads 2L, 2L+1)
#pragma unroll
                    for (int step = 0; step < 5; ++step) {
                        const int o = 16 >> step;
                        const int wdt = 32 >> step;  // heads kept after this step
                        const bool upper = (lane & o) != 0;
#pragma unroll
                        for (int k = 0; k < wdt; ++k) {
                            const float sm = upper ? m[k] : m[k + wdt], sl = upper ? ls[k] : ls[k + wdt];
                            float km = upper ? m[k + wdt] : m[k], kl = upper ? ls[k + wdt] : ls[k];
                            const float rm = __shfl_xor_sync(0xffffffffu, sm, o);
                            const float rl = __shfl_xor_sync(0xffffffffu, sl, o);
                            const float mm = fmaxf(km, rm);
                            if (mm != -INFINITY) {
                                kl = kl * ex2_approx(km - mm) + rl * ex2_approx(rm - mm);
                                km = mm;
                            }
                            m[k] = km;
                            ls[k] = kl;
                        }
                    }
                    float* red = red_s + warp * 128;
                    red[4 * lane + 0] = m[0];
                    red[4 * lane + 1] = ls[0];
                    red[4 * lane + 2] = m[1];
                    red[4 * lane + 3] = ls[1];
                    named_bar_sync(1, 128);
                    if (tid < 64) {
                        float mm = -INFINITY, ll = 0.f;
                        for (int w = 0; w < 4; ++w) {
                            const float m2 = red_s[w * 128 + 2 * tid], l2 = red_s[w * 128 + 2 * tid + 1];
                            const float mx = fmaxf(mm, m2);
                            if (mx != -INFINITY) {
                                ll = ll * ex2_approx(mm - mx) + l2 * ex2_approx(m2 - mx);
                                mm = mx;
                            }
                        }
                        hm_s[tid] = mm;
                        hl_s[tid] = ll > 0.f ? 1.f / ll : 0.f;
                    }
                    named_bar_sync(1, 128);
                    // ---- probability pass: resident tiles from tensor memory, then
                    // the spilled ones from the workspace (the next tile's loads in
                    // flight while one is summed)
                    // sum over heads g0 .. g0+31 of 2^(z - max) / sum; z4(i) gives
                    // the logits of heads g0 + 4i .. g0 + 4i + 3
                    auto prob_sum = [&](auto&& z4, int g0, float acc) {
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            const float4 z = z4(i);
                            const float4 hm = *reinterpret_cast<const float4*>(hm_s + g0 + 4 * i);
                            const float4 hl = *reinterpret_cast<const float4*>(hl_s + g0 + 4 * i);
                            acc = fmaf(ex2_approx(fmaf(z.x, c_log2, -hm.x)), hl.x, acc);
                            acc = fmaf(ex2_approx(fmaf(z.y, c_log2, -hm.y)), hl.y, acc);
                            acc = fmaf(ex2_approx(fmaf(z.z, c_log2, -hm.z)), hl.z, acc);
                            acc = fmaf(ex2_approx(fmaf(z.w, c_log2, -hm.w)), hl.w, acc);
                        }
                        return acc;
                    };
                    for (int t = R; t < T; ++t) {
                        const uint32_t j = job0 + t;
                        const uint32_t ta = tmem_base + lane_base + static_cast<uint32_t>(j % NSLOT) * 64;
                        float acc = 0.f;
#pragma unroll
                        for (int half = 0; half < 2; ++half) {
                            uint32_t v[32];
                            tmem_ld<32>(ta + half * 32, v);
                            tmem_wait_ld();
                            acc = prob_sum(
                                [&](int i) {
                                    return make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                                       __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
                                },
                                half * 32, acc);
                        }
                        release(j);
                        const int slot = t * Cfg::BM + tid;
                        if (slot < n) P_s[slot] += acc * inv_norm;
                    }
                    if (R > 0) {
                        // half tiles (32 heads, 8 float4) in order, each loaded one
                        // half ahead of its sum
                        float4 cur[8];
#pragma unroll
                        for (int g = 0; g < 8; ++g) cur[g] = spill[g * Cfg::BM + tid];
                        for (int t = 0; t < R; ++t) {
                            const float4* sp = spill + static_cast<size_t>(t) * 16 * Cfg::BM + tid;
                            float4 nxt[8];
#pragma unroll
                            for (int g = 0; g < 8; ++g) nxt[g] = sp[(8 + g) * Cfg::BM];
                            float acc = prob_sum([&](int i) { return cur[i]; }, 0, 0.f);
                            if (t + 1 < R) {
#pragma unroll
                                for (int g = 0; g < 8; ++g) cur[g] = sp[(16 + g) * Cfg::BM];
                            }
                            acc = prob_sum([&](int i) { return nxt[i]; }, 32, acc);
                            const int slot = t * Cfg::BM + tid;
                            if (slot < n) P_s[slot] += acc * inv_norm;
                        }
                    }
                    job = job0 + T;
                }
                // ---- the indexer's scores of the same keys
                for (int t = 0; t < T; ++t) {
                    const uint32_t ta = acquire(job);
                    float score = 0.f;
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        uint32_t v[32];
                        tmem_ld<32>(ta + half * 32, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int k = 0; k < 32; k += 4) {
                            const float4 wv = *reinterpret_cast<const float4*>(w_s + half * 32 + k);
                            score = fmaf(wv.x, fmaxf(__uint_as_float(v[k + 0]), 0.f), score);
                            score = fmaf(wv.y, fmaxf(__uint_as_float(v[k + 1]), 0.f), score);
                            score = fmaf(wv.z, fmaxf(__uint_as_float(v[k + 2]), 0.f), score);
                            score = fmaf(wv.w, fmaxf(__uint_as_float(v[k + 3]), 0.f), score);
                        }
                    }
                    release(job);
                    ++job;
                    const int slot = t * Cfg::BM + tid;
                    if (slot < n) {
                        if (p.k_scale) score *= p.k_scale[static_cast<int64_t>(b) * p.n_k + list_s[buf * Cfg::MAX_TOPK + slot]];
                        Z_s[slot] = score;
                    }
                }
            }
            named_bar_sync(1, 128);  // P and Z complete
            // ---- softmax of the scores and the KL (block reductions over the slots)
            float zmax = -INFINITY;
            for (int i = tid; i < n; i += 128) zmax = fmaxf(zmax, Z_s[i]);
            for (int o = 16; o > 0; o >>= 1) zmax = fmaxf(zmax, __shfl_xor_sync(0xffffffffu, zmax, o));
            if (lane == 0) red_s[warp] = zmax;
            named_bar_sync(1, 128);
            zmax = fmaxf(fmaxf(red_s[0], red_s[1]), fmaxf(red_s[2], red_s[3]));
            named_bar_sync(1, 128);
            float esum = 0.f;
            for (int i = tid; i < n; i += 128) esum += expf(Z_s[i] - zmax);
            for (int o = 16; o > 0; o >>= 1) esum += __shfl_xor_sync(0xffffffffu, esum, o);
            if (lane == 0) red_s[warp] = esum;
            named_bar_sync(1, 128);
            esum = (red_s[0] + red_s[1]) + (red_s[2] + red_s[3]);
            named_bar_sync(1, 128);
            const float log_z = zmax + logf(esum);
            float part = 0.f;
            for (int i = tid; i < n; i += 128) {
                const float pj = P_s[i];
                if (pj > 0.f) part += pj * (logf(pj) - (Z_s[i] - log_z));
            }
            for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
            if (lane == 0) red_s[warp] = part;
            named_bar_sync(1, 128);
            if (tid == 0) p.kl[row] = n > 0 ? (red_s[0] + red_s[1]) + (red_s[2] + red_s[3]) : 0.f;
            // ---- the target row at the index row's positions (the same ordered
            // compaction as the producers': slot = rank among the valid entries)
            if (p.target) {
                const int32_t* irow = p.idx + static_cast<int64_t>(row) * p.topk;
                float* trow = p.target + static_cast<int64_t>(row) * p.topk;
                int run = 0;
                for (int e0 = 0; e0 < p.topk; e0 += 128) {
                    const int e = e0 + tid;
                    const int s = e < p.topk ? irow[e] : -1;
                    const bool ok = s >= 0 && s < p.n_k;
                    const uint32_t bal = __ballot_sync(0xffffffffu, ok);
                    named_bar_sync(1, 128);  // the previous chunk's counts are read
                    if (lane == 0) misc_s[24 + warp] = __popc(bal);
                    named_bar_sync(1, 128);
                    int before = 0, total = 0;
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        const int c = misc_s[24 + w];
                        before += w < warp ? c : 0;
                        total += c;
                    }
                    if (e < p.topk) {
                        const int slot = run + before + __popc(bal & lanemask_lt());
                        trow[e] = (ok && IC_DCHECK(slot < n)) ? P_s[slot] : 0.f;
                    }
                    run += total;
                }
            }
            named_bar_sync(1, 128);  // every read of the list, P and Z is done
            if (tid == 0) mbar_arrive(bar_list_free(buf));
        }
    }

    // ---------------------------------------------------------------- teardown
    __syncthreads();
    if (*abort_flag) {
        if (warp == MMA_WARP && lane == 0) {
            mma_commit(bar_drain);
            mbar_drain(bar_drain, 0);
        }
        __syncthreads();
    }
    if (warp == MMA_WARP) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

}  // namespace ic
