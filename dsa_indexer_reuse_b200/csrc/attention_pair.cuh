// Sparse attention with paired score tiles, for the 576 / 512 latent shape.
//
// What it computes is what sparse_attn_kernel computes (IndexCache paper,
// Abstract: core attention over the k selected tokens): for every query row
// and head h, out[h,:] = sum_{s in idx} softmax_s(sm_scale q[h,:] . kv[s,:576]) kv[s,:512].
//
// Why a second kernel: on sm_100a a tcgen05.mma of this operand shape costs
// about the same per instruction whether M is 64 or 128 (the score MMAs of
// sparse_attn_kernel, 36 per 64-key tile at M = 64, issue at ~96 cycles each
// and set the tile period). So the scores of two 64-key tiles are formed by
// one M = 128 MMA chain: the two shared-memory stages are interleaved chunk
// by chunk (chunk c of stage 0, then chunk c of stage 1, 16 KB per chunk
// slot), so rows 0-63 of a 128-row operand are tile 2p and rows 64-127 are
// tile 2p + 1. TMEM lane i of the score accumulator then holds key i of the
// pair, and a softmax thread owns one key and 32 heads (32x32b loads).
//
// Pipeline per pair: scores (36 MMAs, M = 128) -> softmax of both tiles ->
// P.V of tile 2p (stage 0) and of tile 2p + 1 (stage 1), each freeing its
// stage for the gather of the next pair's tile. A row with an odd tile count
// ends with a lone tile in stage 0: its score MMAs still run at M = 128, and
// the 64 lanes of stage 1 (whatever that stage holds) are masked out.
//
// Everything else (fixed per-head softmax reference with the rare rescale,
// P^T written over the tile's rope columns, O^T = V^T . P^T at M = 128 rows
// of d_v, decode splits with partial (m, l, O)) follows sparse_attn_kernel.
#pragma once

#include "attention.cuh"

// setmaxnreg split of the paired kernel (softmax warpgroups / the rest)
#ifndef IC_ATTN_PAIR_REGS_SMX
#define IC_ATTN_PAIR_REGS_SMX 152
#endif

namespace ic {

template <class Cfg>
__global__ void __launch_bounds__(Cfg::THREADS, 1)
    sparse_attn_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kv,
                            const AttnParams p) {
    static_assert(Cfg::DQK == 576 && Cfg::DV == 512 && Cfg::TMA_CH == 0 && Cfg::P_IN_ROPE, "paired tiles: 576 / 512");
    static_assert(IC_ATTN_PAIR_REGS_SMX % 8 == 0 && IC_ATTN_PAIR_REGS_SMX >= 136 && IC_ATTN_PAIR_REGS_SMX <= 176,
                  "register split");
    constexpr int PCH = 2 * Cfg::CH_BYTES;  // one chunk slot: chunk c of both stages
    constexpr uint32_t IDESC_S2 = make_idesc(128, Cfg::NH, FMT_BF16, FMT_BF16);
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align_smem_1024(smem_raw);
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
    auto bar_s_full = [&](int b) { return bar0 + 48u + 8u * b; };
    auto bar_s_free = [&](int b) { return bar0 + 64u + 8u * b; };
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
            mbar_init(bar_kv_full(s), Cfg::NPROD);
            mbar_init(bar_kv_empty(s), 1);
            mbar_init(bar_s_full(s), 1);
            mbar_init(bar_s_free(s), 8);
            mbar_init(bar_p_full(s), 4);  // the four softmax warps holding that stage's keys
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
    // copies issued by the producers' first thread: Q loads armed (count), and
    // per stage the use count of its last armed gather
    uint32_t q_armed = 0, kv_armed[2] = {0u, 0u};

    if (warp >= 8) {
      regs_dec<256 - IC_ATTN_PAIR_REGS_SMX>();
      if (warp != MMA_WARP) {
        // ------------------------------ index compaction + cp.async row gathers
        const int pw = warp < MMA_WARP ? warp - 8 : warp - 9;  // producer warp 0..6
        const int ptid = pw * 32 + lane;
        if (ptid == 0) prefetch_tmap(&tm_q);
        uint32_t ku[2] = {0u, 0u};  // tiles gathered into each stage so far
        uint32_t q_n = 0;
        for (int r = 0; r < n_rounds; ++r) {
            const int item = attn_snake(r, blockIdx.x, gridDim.x);
            if (item >= p.n_work) continue;
            const AttnWork wk = attn_work(p, item);
            const int b = static_cast<int>(wk.row / p.n_q);
            // compact the valid entries of the index row, keeping their order
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
                    const int s = j & 1;  // tile j of a row lives in stage j % 2
                    // warp pw takes rows pw, pw+NW, ...; their source rows are looked
                    // up before the wait for the stage, off the refill's critical path
                    constexpr int NW = Cfg::NPROD / 32;
                    constexpr int RPW = (Cfg::BK + NW - 1) / NW;  // rows per warp
                    constexpr int UPR = Cfg::NCH * 8;
                    constexpr int UPL = (UPR + 31) / 32;
                    const __nv_bfloat16* src[RPW];
#pragma unroll
                    for (int i = 0; i < RPW; ++i) {
                        const int rr = pw + NW * i;
                        const int e = lo + j * Cfg::BK + rr;
                        int key = (rr < Cfg::BK && e < hi) ? list_s[e] : fallback;
                        if (!IC_DCHECK(key >= 0 && key < p.n_k)) key = 0;
                        src[i] = kvb + static_cast<int64_t>(key) * Cfg::DQK;
                    }
                    if (mbar_wait(bar_kv_empty(s), (ku[s] & 1) ^ 1, abort_flag)) {
                        kv_armed[s] = ku[s] + 1;
                        // a row's 72 16-byte units go to its chunk slots, 128-byte swizzled
                        const uint32_t stage = s_base + Cfg::OFF_T + s * Cfg::CH_BYTES;
#pragma unroll
                        for (int i = 0; i < RPW; ++i) {
                            const int rr = pw + NW * i;
                            if (rr >= Cfg::BK) break;
                            const uint32_t row_dst = stage + (rr >> 3) * 1024 + (rr & 7) * 128;
                            const int x = rr & 7;
#pragma unroll
                            for (int k = 0; k < UPL; ++k) {
                                const int u = lane + 32 * k;
                                if (u < UPR)
                                    cp_async_16(row_dst + (u >> 3) * PCH + (((u & 7) ^ x) << 4), src[i] + u * 8);
                            }
                        }
                        cp_async_mbar_arrive_noinc(bar_kv_full(s));
                    }
                    ++ku[s];
                }
                ++q_n;
            }
            // list_s and cnt_s are rewritten by the next row's compaction
            named_bar_sync(3, Cfg::NPROD);
        }
      } else {
        // ------------------------------------------------------------ MMA issuer
        uint32_t ku[2] = {0u, 0u};  // tiles consumed from each stage so far
        uint32_t pc = 0, q_n = 0;   // pairs so far (score buffer parity), rows so far
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
                const int n_pairs = (n_tiles + 1) >> 1;
                for (int pp = 0; pp < n_pairs; ++pp) {
                    const int nt = 2 * pp + 1 < n_tiles ? 2 : 1;  // tiles in this pair
                    // ---- S^T of the pair = K_pair . Q^T, one M = 128 chain
                    bool go = mbar_wait(bar_kv_full(0), ku[0] & 1, abort_flag);
                    if (nt == 2) go = mbar_wait(bar_kv_full(1), ku[1] & 1, abort_flag) && go;
                    fence_proxy_async_smem();  // cp.async-written chunks before the MMA reads
                    const int sb = pc & 1;
                    go = mbar_wait(bar_s_free(sb), ((pc >> 1) & 1) ^ 1, abort_flag) && go;
                    tc_fence_after();
                    if (go) {
                        const uint64_t adesc0 = make_sw128_desc(s_base + Cfg::OFF_T);
                        const uint64_t bdesc0 = make_sw128_desc(s_base + Cfg::OFF_Q);
                        const uint32_t d_s = tmem_base + Cfg::S_COL + 64 * sb;
#pragma unroll
                        for (int ch = 0; ch < Cfg::NCH; ++ch) {
#pragma unroll
                            for (int k4 = 0; k4 < 4; ++k4) {
                                const int ks = ch * 4 + k4;
                                const uint32_t a_off = (ch * PCH + k4 * 32) >> 4;
                                const uint32_t b_off = (ch * Cfg::Q_CH_BYTES + k4 * 32) >> 4;
                                mma_f16(d_s, adesc0 + a_off, bdesc0 + b_off, IDESC_S2, ks > 0 ? 1u : 0u);
                            }
                        }
                        mma_commit(bar_s_full(sb));
                        if (pp == n_pairs - 1) mma_commit(bar_q_empty);
                    }
                    ++pc;
                    // ---- O^T += V^T . P^T for the pair's tiles, each freeing its stage
                    for (int s = 0; s < nt; ++s) {
                        const bool first = pp == 0 && s == 0;
                        bool ok = go && mbar_wait(bar_p_full(s), ku[s] & 1, abort_flag);
                        if (first) ok = ok && mbar_wait(bar_o_free, (q_n & 1) ^ 1, abort_flag);
                        tc_fence_after();
                        if (ok) {
                            const uint32_t stage = s_base + Cfg::OFF_T + s * Cfg::CH_BYTES;
                            const uint64_t adesc0 = make_sw128_desc(stage, PCH, 1024);
                            const uint64_t bdesc0 = make_sw128_desc(stage + Cfg::P_CHUNK * PCH, PCH, 1024);
#pragma unroll
                            for (int vb = 0; vb < Cfg::NVB; ++vb) {
#pragma unroll
                                for (int ks = 0; ks < Cfg::BK / 16; ++ks) {
                                    const uint32_t a_off = ((vb * Cfg::VB_M / 64) * PCH + ks * 2048) >> 4;
                                    mma_f16(tmem_base + Cfg::O_COL + 64 * vb, adesc0 + a_off,
                                            bdesc0 + ((ks * 2048) >> 4), Cfg::IDESC_O, (first && ks == 0) ? 0u : 1u);
                                }
                            }
                            mma_commit(bar_kv_empty(s));
                        }
                        go = ok;
                    }
                    if (go) mma_commit(bar_pv_done);
                    ++ku[0];
                    if (nt == 2) ++ku[1];
                }
            }
            __syncwarp();
            ++q_n;
        }
      }
    } else {
        regs_inc<IC_ATTN_PAIR_REGS_SMX>();
        // ------------------------------------------------- softmax and output
        const int wq = warp & 3;               // TMEM lane quarter: keys 32 wq .. 32 wq + 31 of a pair
        const int sw = warp >> 2;              // softmax warpgroup
        const int hb = Cfg::SMX_HEADS * sw;    // its heads: [hb, hb + 32)
        const int wtid = threadIdx.x - 128 * sw;
        const int sbar = 1 + sw;               // its named barrier
        const int ps = wq >> 1;                // stage of this thread's key
        const int key_in_tile = (wq & 1) * 32 + lane;
        uint32_t pc = 0;  // pairs handled so far
        for (int r = 0; r < n_rounds; ++r) {
            const int item = attn_snake(r, blockIdx.x, gridDim.x);
            if (item >= p.n_work) continue;
            const AttnWork wk = attn_work(p, item);
            const int n_valid = warp_count_valid(p.idx + wk.row * p.topk, p.topk, p.n_k, lane);
            const int len = ceil_div(ceil_div(n_valid, p.n_splits), Cfg::BK) * Cfg::BK;
            const int lo = min(n_valid, wk.split * len);
            const int hi = min(n_valid, lo + len);
            const int n_tiles = ceil_div(hi - lo, Cfg::BK);
            const int n_pairs = (n_tiles + 1) >> 1;

            float l_part[32];
#pragma unroll
            for (int c = 0; c < 32; ++c) l_part[c] = 0.f;

            for (int pp = 0; pp < n_pairs; ++pp) {
                const int sb = pc & 1;
                mbar_wait(bar_s_full(sb), (pc >> 1) & 1, abort_flag);
                tc_fence_after();
                uint32_t sv[32];
                tmem_ld<32>(tmem_base + (static_cast<uint32_t>(wq * 32) << 16) + Cfg::S_COL + 64 * sb + hb, sv);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_s_free(sb));
                const int tile = 2 * pp + ps;
                const bool has_tile = tile < n_tiles;  // uniform across the warp
                const bool valid = lo + tile * Cfg::BK + key_in_tile < hi;
                if (pp == 0) {
                    // reference logit per head: the first key of this slice
                    if (wq == 0 && lane == 0) {
#pragma unroll
                        for (int c = 0; c < 32; ++c) m_s[hb + c] = __fmul_rn(__uint_as_float(sv[c]), p.sm_scale_log2);
                    }
                    named_bar_sync(sbar, 128);
                }
                // z = logit (log2 units) minus the per-head reference, in place
                float zmax = -INFINITY;
#pragma unroll
                for (int c = 0; c < 32; c += 4) {
                    const float4 m4 = *reinterpret_cast<const float4*>(m_s + hb + c);
                    const float z0 = fmaf(__uint_as_float(sv[c + 0]), p.sm_scale_log2, -m4.x);
                    const float z1 = fmaf(__uint_as_float(sv[c + 1]), p.sm_scale_log2, -m4.y);
                    const float z2 = fmaf(__uint_as_float(sv[c + 2]), p.sm_scale_log2, -m4.z);
                    const float z3 = fmaf(__uint_as_float(sv[c + 3]), p.sm_scale_log2, -m4.w);
                    zmax = fmaxf(zmax, fmaxf(fmaxf(z0, z1), fmaxf(z2, z3)));
                    sv[c + 0] = __float_as_uint(z0);
                    sv[c + 1] = __float_as_uint(z1);
                    sv[c + 2] = __float_as_uint(z2);
                    sv[c + 3] = __float_as_uint(z3);
                }
                if (!valid) zmax = -INFINITY;
                if (named_bar_or(sbar, 128, zmax > IC_ATTN_RESCALE_LOG2)) {
                    // rare path: raise the reference to the pair's maximum and
                    // rescale the accumulated output and row sums. Every P.V issued
                    // so far for this row is complete: the pair's scores were
                    // issued after them and are in hand.
                    float t[32];
#pragma unroll
                    for (int c = 0; c < 32; ++c) t[c] = valid ? __uint_as_float(sv[c]) : -INFINITY;
                    // butterfly over the warp's keys: lane L ends with head hb + L
#pragma unroll
                    for (int step = 0; step < 5; ++step) {
                        const int o = 16 >> step;
                        const bool upper = (lane & o) != 0;
#pragma unroll
                        for (int k = 0; k < o; ++k) {
                            const float send = upper ? t[k] : t[k + o];
                            const float keep = upper ? t[k + o] : t[k];
                            t[k] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, o));
                        }
                    }
                    red_s[wq * 64 + hb + lane] = t[0];
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
                    for (int c = 0; c < 32; ++c) {
                        const float dz = a_s[hb + c];
                        l_part[c] *= ex2_approx(-dz);
                        sv[c] = __float_as_uint(__uint_as_float(sv[c]) - dz);
                    }
                    if (pp >= 1) {
                        for (int vb = 0; vb < Cfg::NVB; ++vb) {
                            uint32_t o32[32];
                            const uint32_t ta =
                                tmem_base + (static_cast<uint32_t>(wq * 32) << 16) + Cfg::O_COL + 64 * vb + 32 * sw;
                            tmem_ld<32>(ta, o32);
                            tmem_wait_ld();
#pragma unroll
                            for (int c = 0; c < 32; ++c)
                                o32[c] = __float_as_uint(__uint_as_float(o32[c]) * ex2_approx(-a_s[32 * sw + c]));
                            tmem_st32(ta, o32);
                        }
                        tmem_wait_st();
                    }
                    named_bar_sync(sbar, 128);
                }
                // probabilities, row sums, and this key's bf16 P^T row (heads hb .. hb+31)
                uint32_t packed[16];
                if (valid) {  // uniform per thread: only a slice's last tile has invalid keys
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float p0 = ex2_approx(__uint_as_float(sv[2 * i]));
                        const float p1 = ex2_approx(__uint_as_float(sv[2 * i + 1]));
                        l_part[2 * i] += p0;
                        l_part[2 * i + 1] += p1;
                        packed[i] = pack_bf16x2(p0, p1);
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 16; ++i) packed[i] = 0u;
                }
                if (has_tile) {
                    const uint32_t prow = s_base + Cfg::OFF_T + Cfg::P_CHUNK * PCH + ps * Cfg::CH_BYTES +
                                          (key_in_tile >> 3) * 1024 + (key_in_tile & 7) * 128;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int u = hb / 8 + i;
                        st_shared_v4(prow + ((u ^ (key_in_tile & 7)) << 4), packed[4 * i], packed[4 * i + 1],
                                     packed[4 * i + 2], packed[4 * i + 3]);
                    }
                    fence_proxy_async_smem();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bar_p_full(ps));
                }
                ++pc;
            }

            // ---- end of row: row sums, then the output (or the partials), once
            // the row's last P.V products are complete (their pair's barrier
            // phase is the only one outstanding: the pair before completed
            // before this pair's scores were issued)
            if (n_tiles > 0) {
                mbar_wait(bar_pv_done, (pc - 1) & 1, abort_flag);
                tc_fence_after();
            }
            // butterfly over the warp's keys: lane L ends with head hb + L
#pragma unroll
            for (int step = 0; step < 5; ++step) {
                const int o = 16 >> step;
                const bool upper = (lane & o) != 0;
#pragma unroll
                for (int k = 0; k < o; ++k) {
                    const float send = upper ? l_part[k] : l_part[k + o];
                    const float keep = upper ? l_part[k + o] : l_part[k];
                    l_part[k] = keep + __shfl_xor_sync(0xffffffffu, send, o);
                }
            }
            red_s[wq * 64 + hb + lane] = l_part[0];
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
                const int v = vb * Cfg::VB_M + wq * 32 + lane;
                uint32_t o32[32];
                if (n_tiles > 0) {
                    tmem_ld<32>(tmem_base + (static_cast<uint32_t>(wq * 32) << 16) + Cfg::O_COL + 64 * vb + 32 * sw,
                                o32);
                    tmem_wait_ld();
                } else {
#pragma unroll
                    for (int c = 0; c < 32; ++c) o32[c] = 0u;
                }
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const int h = 32 * sw + c;
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
                for (int s = 0; s < 2; ++s)
                    if (kv_armed[s] > 0) mbar_drain(bar_kv_full(s), (kv_armed[s] - 1) & 1);
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

}  // namespace ic
