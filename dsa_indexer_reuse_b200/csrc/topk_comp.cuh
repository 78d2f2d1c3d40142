// Exact top-k selection over unordered candidate lists, for sm_100a.
//
// Selection rule (IndexCache paper, Abstract: the indexer "selects the top-k
// most relevant tokens per query"; ties go to the lower key index): a
// candidate (key, index), where `key` is the order-preserving unsigned image
// of its fp32 score, is ranked by the 64-bit composite
//     comp = key << 32 | ~index,
// so a higher score wins and, at equal scores, the lower index wins. The
// composites of distinct keys are distinct, so every cut of a list is a
// single threshold: "keep comp > tau" (or ">= tau"), with no tie handling.
// Lists that carry the composite order need no position order, which lets
// the epilogue warps append without a barrier (shared-memory atomics).
//
// Layout of a list of n entries among NT threads: position e = m * NT + t
// lives in thread t, round m (consecutive lanes read consecutive words).
// Compaction is stable (the kept entries keep their relative list order),
// so any order a producer establishes within a subset of the list (for
// example ascending indices per appending warp) survives every cut.
#pragma once

#include "common.cuh"
#include "topk_select.cuh"

namespace ic {

__device__ __forceinline__ uint64_t comp_key(uint32_t key, int32_t idx) {
    return (static_cast<uint64_t>(key) << 32) | static_cast<uint64_t>(~static_cast<uint32_t>(idx));
}

__device__ __forceinline__ uint64_t shfl_xor64(uint64_t v, int m) {
    const uint32_t lo = __shfl_xor_sync(0xffffffffu, static_cast<uint32_t>(v), m);
    const uint32_t hi = __shfl_xor_sync(0xffffffffu, static_cast<uint32_t>(v >> 32), m);
    return (static_cast<uint64_t>(hi) << 32) | lo;
}

__device__ __forceinline__ uint64_t shfl64(uint64_t v, int src) {
    const uint32_t lo = __shfl_sync(0xffffffffu, static_cast<uint32_t>(v), src);
    const uint32_t hi = __shfl_sync(0xffffffffu, static_cast<uint32_t>(v >> 32), src);
    return (static_cast<uint64_t>(hi) << 32) | lo;
}

// One warp sorts 32 composites descending (bitonic); lane r ends with rank r.
// Empty slots carry 0 and sort last.
__device__ __forceinline__ uint64_t warp_sort_desc64(uint64_t v, int lane) {
#pragma unroll
    for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            const uint64_t o = shfl_xor64(v, stride);
            const bool lower = (lane & stride) == 0;
            const bool desc = (size == 32) || ((lane & size) == 0);
            // in a descending block the lower lane keeps the larger value
            const bool take = (lower == desc) ? (o > v) : (o < v);
            if (take) v = o;
        }
    }
    return v;
}

__device__ __forceinline__ uint64_t warp_or64(uint64_t v) {
    const uint32_t lo = __reduce_or_sync(0xffffffffu, static_cast<uint32_t>(v));
    const uint32_t hi = __reduce_or_sync(0xffffffffu, static_cast<uint32_t>(v >> 32));
    return (static_cast<uint64_t>(hi) << 32) | lo;
}

// Scratch of the composite selection (per cooperating group).
template <int NT, int E>
struct CompScratch {
    static_assert(NT % 32 == 0 && NT <= 1024, "NT");
    static_assert(E >= 1 && E <= 32, "E");
    static constexpr int NW = NT / 32;
    static constexpr int NG = 4;                 // output groups of the grouped emit
    static constexpr int NTBL = NG * E * NW;     // (group, round, warp) count table
    // the selection's histogram and the count table of the compaction /
    // emission are never live at the same time
    union {
        int hist[256];
        int tbl[NTBL > 256 ? NTBL : 256];
    };
    uint64_t g64[64];      // boundary-bucket gather
    uint64_t wref[NW];     // per-warp reference / OR of differences
    uint32_t rmin[NW], rmax[NW];
    int red[NW];
    int scan_tmp[2][NW];
    int misc[8];
    uint64_t tau;
};

// Number of list positions p < n with pred(p). Contains two barriers.
template <int NT, int E, class Pred>
__device__ __forceinline__ int comp_block_count(int n, int tid, int bar_id, CompScratch<NT, E>& sc, Pred&& pred) {
    constexpr int NW = NT / 32;
    const int lane = tid & 31, warp = tid >> 5;
    int c = 0;
#pragma unroll 8
    for (int m = 0; m < E; ++m) {
        const int pos = m * NT + tid;
        if (pos < n && pred(pos)) ++c;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    if (lane == 0) sc.red[warp] = c;
    named_bar_sync(bar_id, NT);
    int total = 0;
#pragma unroll
    for (int w = 0; w < NW; ++w) total += sc.red[w];
    named_bar_sync(bar_id, NT);  // sc.red is free again
    return total;
}

// Fallback of comp_select_kth (same contract): a 256-bucket histogram in
// value space (between the list's minimum and maximum score) finds the
// bucket of the k-th best; a bucket of at most 32 entries is sorted by one
// warp, a larger one is resolved by an MSB-first radix select over the
// composites of its entries, starting at the highest bit in which they differ.
template <int NT, int E, class LoadKey, class LoadId>
__device__ uint64_t comp_select_kth_radix(int n, int k, int tid, int bar_id, CompScratch<NT, E>& sc,
                                          LoadKey&& load_key, LoadId&& load_id) {
    constexpr int NW = NT / 32;
    const int lane = tid & 31, warp = tid >> 5;
    auto valid = [&](int m) { return m * NT + tid < n; };

    uint32_t kmin = 0xffffffffu, kmax = 0u;
#pragma unroll 8
    for (int m = 0; m < E; ++m) {
        if (valid(m)) {
            const uint32_t km = load_key(m * NT + tid);
            kmin = min(kmin, km);
            kmax = max(kmax, km);
        }
    }
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    for (int i = tid; i < 256; i += NT) sc.hist[i] = 0;
    if (lane == 0) {
        sc.rmin[warp] = kmin;
        sc.rmax[warp] = kmax;
    }
    named_bar_sync(bar_id, NT);
    kmin = 0xffffffffu;
    kmax = 0u;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
        kmin = min(kmin, sc.rmin[w]);
        kmax = max(kmax, sc.rmax[w]);
    }
    // value buckets; when every score is equal, one bucket holds everything
    const float lo_f = ordered_to_float(kmin);
    const float span = ordered_to_float(kmax) - lo_f;
    const float scale_f =
        (kmin != kmax && isfinite(span) && span > 0.f && isfinite(256.0f / span)) ? 256.0f / span : 0.f;
#pragma unroll 8
    for (int m = 0; m < E; ++m)
        if (valid(m)) atomicAdd(&sc.hist[value_bin(load_key(m * NT + tid), lo_f, scale_f)], 1);
    named_bar_sync(bar_id, NT);
    if (warp == 0) {
        int c[8];
        int local = 0;
#pragma unroll
        for (int b = 0; b < 8; ++b) {
            c[b] = sc.hist[8 * lane + b];
            local += c[b];
        }
        int suffix = local;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int v = __shfl_down_sync(0xffffffffu, suffix, off);
            if (lane + off < 32) suffix += v;
        }
        const int above = suffix - local;
        if (above < k && k <= suffix) {
            int cum = above;
#pragma unroll
            for (int b = 7; b >= 0; --b) {
                if (cum < k && k <= cum + c[b]) {
                    sc.misc[1] = 8 * lane + b;
                    sc.misc[2] = cum;
                    sc.misc[3] = c[b];
                }
                cum += c[b];
            }
        }
        if (lane == 0) sc.misc[0] = 0;  // gather counter
    }
    named_bar_sync(bar_id, NT);
    const int dstar = sc.misc[1];
    const int need = k - sc.misc[2];  // rank of the answer within the bucket, 1-based
    const int in_bin = sc.misc[3];
    auto in_bucket = [&](int m, uint32_t km) { return valid(m) && value_bin(km, lo_f, scale_f) == dstar; };

    if (in_bin <= 32) {
#pragma unroll
        for (int m = 0; m < E; ++m) {
            const int pos = m * NT + tid;
            const uint32_t km = valid(m) ? load_key(pos) : 0u;
            if (in_bucket(m, km)) {
                const int slot = atomicAdd(&sc.misc[0], 1);
                if (slot < 32) sc.g64[slot] = comp_key(km, load_id(pos));
            }
        }
        named_bar_sync(bar_id, NT);
        if (warp == 0) {
            const uint64_t v = warp_sort_desc64(lane < in_bin ? sc.g64[lane] : 0ull, lane);
            if (lane == need - 1) sc.tau = v;
        }
        named_bar_sync(bar_id, NT);
        const uint64_t tau = sc.tau;
        named_bar_sync(bar_id, NT);  // sc.tau may be rewritten by the caller
        return tau;
    }

    // crowded bucket: radix select over the composites of its entries
    uint64_t ref = 0;
    bool have = false;
#pragma unroll
    for (int m = 0; m < E; ++m) {
        const int pos = m * NT + tid;
        const uint32_t km = valid(m) ? load_key(pos) : 0u;
        if (!have && in_bucket(m, km)) {
            ref = comp_key(km, load_id(pos));
            have = true;
        }
    }
    const uint32_t bal = __ballot_sync(0xffffffffu, have);
    const uint64_t wr = shfl64(ref, bal ? __ffs(bal) - 1 : 0);
    if (lane == 0) {
        sc.wref[warp] = wr;
        sc.red[warp] = bal != 0;
    }
    named_bar_sync(bar_id, NT);
#pragma unroll
    for (int w = NW - 1; w >= 0; --w)
        if (sc.red[w]) ref = sc.wref[w];
    named_bar_sync(bar_id, NT);  // wref and red are reused below
    uint64_t diff = 0;
#pragma unroll
    for (int m = 0; m < E; ++m) {
        const int pos = m * NT + tid;
        const uint32_t km = valid(m) ? load_key(pos) : 0u;
        if (in_bucket(m, km)) diff |= comp_key(km, load_id(pos)) ^ ref;
    }
    diff = warp_or64(diff);
    if (lane == 0) sc.wref[warp] = diff;
    named_bar_sync(bar_id, NT);
    diff = 0;
#pragma unroll
    for (int w = 0; w < NW; ++w) diff |= sc.wref[w];
    // in_bin > 32 distinct composites differ somewhere
    int hb = 63 - __clzll(static_cast<long long>(diff | 1ull));
    uint64_t pmask = (hb == 63) ? 0ull : ~((2ull << hb) - 1ull);
    uint64_t prefix = ref & pmask;
    int remaining = need;
    while (true) {
        const int shift = hb >= 7 ? hb - 7 : 0;
        const int width = hb - shift + 1;
        const uint64_t dmask = (1ull << width) - 1ull;
        for (int i = tid; i < 256; i += NT) sc.hist[i] = 0;
        named_bar_sync(bar_id, NT);
#pragma unroll
        for (int m = 0; m < E; ++m) {
            const int pos = m * NT + tid;
            const uint32_t km = valid(m) ? load_key(pos) : 0u;
            if (in_bucket(m, km)) {
                const uint64_t cv = comp_key(km, load_id(pos));
                if ((cv & pmask) == prefix) atomicAdd(&sc.hist[static_cast<int>((cv >> shift) & dmask)], 1);
            }
        }
        named_bar_sync(bar_id, NT);
        if (warp == 0) {
            int c[8];
            int local = 0;
#pragma unroll
            for (int b = 0; b < 8; ++b) {
                c[b] = sc.hist[8 * lane + b];
                local += c[b];
            }
            int suffix = local;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int v = __shfl_down_sync(0xffffffffu, suffix, off);
                if (lane + off < 32) suffix += v;
            }
            const int above2 = suffix - local;
            if (above2 < remaining && remaining <= suffix) {
                int cum = above2;
#pragma unroll
                for (int b = 7; b >= 0; --b) {
                    if (cum < remaining && remaining <= cum + c[b]) {
                        sc.misc[4] = 8 * lane + b;
                        sc.misc[5] = cum;
                    }
                    cum += c[b];
                }
            }
        }
        named_bar_sync(bar_id, NT);
        prefix |= static_cast<uint64_t>(sc.misc[4]) << shift;
        pmask |= dmask << shift;
        remaining -= sc.misc[5];
        named_bar_sync(bar_id, NT);  // misc and hist are rewritten by the next pass
        if (shift == 0) break;
        hb = shift - 1;
    }
    return prefix;
}

// One warp sorts the 64 composites at v descending (bitonic in shared memory).
__device__ __forceinline__ void warp_sort64_desc(uint64_t* v, int lane) {
#pragma unroll 1
    for (int size = 2; size <= 64; size <<= 1) {
#pragma unroll 1
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            __syncwarp();
            // the lane-th pair (i, i + stride) with bit `stride` clear in i
            const int i = ((lane & ~(stride - 1)) << 1) | (lane & (stride - 1));
            const int j = i | stride;
            const uint64_t a = v[i], b = v[j];
            const bool desc = (i & size) == 0;
            if (desc ? (a < b) : (a > b)) {
                v[i] = b;
                v[j] = a;
            }
        }
    }
    __syncwarp();
}

// Exact k-th best composite among list positions [0, n), for n > k >= 1.
// All NT threads call it with the same arguments; the result is the same in
// every thread. A radix select over the score keys relative to the list's
// minimum, MSB first in 8-bit digits starting at the highest bit in which
// the keys differ, narrows the candidates to the bucket of the k-th best;
// once that bucket holds at most 64 entries they are gathered and sorted by
// one warp by composite (so equal scores resolve by index). A bucket of more
// than 64 entries with one score (many exact ties) falls back to
// comp_select_kth_radix.
template <int NT, int E, class LoadKey, class LoadId>
__device__ uint64_t comp_select_kth(int n, int k, int tid, int bar_id, CompScratch<NT, E>& sc,
                                    LoadKey&& load_key, LoadId&& load_id) {
    constexpr int NW = NT / 32;
    const int lane = tid & 31, warp = tid >> 5;
    uint32_t kmin = 0xffffffffu, kmax = 0u;
#pragma unroll 8
    for (int m = 0; m < E; ++m) {
        const int pos = m * NT + tid;
        if (pos < n) {
            const uint32_t km = load_key(pos);
            kmin = min(kmin, km);
            kmax = max(kmax, km);
        }
    }
    kmin = __reduce_min_sync(0xffffffffu, kmin);
    kmax = __reduce_max_sync(0xffffffffu, kmax);
    if (lane == 0) {
        sc.rmin[warp] = kmin;
        sc.rmax[warp] = kmax;
    }
    named_bar_sync(bar_id, NT);
    kmin = 0xffffffffu;
    kmax = 0u;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
        kmin = min(kmin, sc.rmin[w]);
        kmax = max(kmax, sc.rmax[w]);
    }
    const uint32_t span = kmax - kmin;
    // digits of r = key - kmin: the first covers bits [shift, hb], then 8 bits each
    int hb = span ? 31 - __clz(span) : 0;
    int shift = hb >= 7 ? hb - 7 : 0;
    uint32_t pmask = 0u, prefix = 0u;
    int remaining = k, in_bin = n;
    while (span != 0u) {
        const uint32_t dmask = (hb - shift + 1 >= 32) ? 0xffffffffu : ((1u << (hb - shift + 1)) - 1u);
        for (int i = tid; i < 256; i += NT) sc.hist[i] = 0;
        named_bar_sync(bar_id, NT);
#pragma unroll 8
        for (int m = 0; m < E; ++m) {
            const int pos = m * NT + tid;
            if (pos < n) {
                const uint32_t r = load_key(pos) - kmin;
                if ((r & pmask) == prefix) atomicAdd(&sc.hist[(r >> shift) & dmask], 1);
            }
        }
        named_bar_sync(bar_id, NT);
        if (warp == 0) {
            // digits in descending order (larger key first)
            int c[8];
            int local = 0;
#pragma unroll
            for (int b = 0; b < 8; ++b) {
                c[b] = sc.hist[8 * lane + b];
                local += c[b];
            }
            int suffix = local;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int v = __shfl_down_sync(0xffffffffu, suffix, off);
                if (lane + off < 32) suffix += v;
            }
            const int above = suffix - local;
            if (above < remaining && remaining <= suffix) {
                int cum = above;
#pragma unroll
                for (int b = 7; b >= 0; --b) {
                    if (cum < remaining && remaining <= cum + c[b]) {
                        sc.misc[4] = 8 * lane + b;
                        sc.misc[5] = cum;
                        sc.misc[6] = c[b];
                    }
                    cum += c[b];
                }
            }
        }
        named_bar_sync(bar_id, NT);
        prefix |= static_cast<uint32_t>(sc.misc[4]) << shift;
        pmask |= dmask << shift;
        remaining -= sc.misc[5];
        in_bin = sc.misc[6];
        named_bar_sync(bar_id, NT);  // misc and hist are rewritten below
        if (in_bin <= 64 || shift == 0) break;
        hb = shift - 1;
        shift = hb >= 7 ? hb - 7 : 0;
    }
    if (in_bin > 64) return comp_select_kth_radix<NT, E>(n, k, tid, bar_id, sc, load_key, load_id);
    // gather the bucket (r & pmask == prefix) and sort it by composite
    if (tid == 0) sc.misc[0] = 0;
    named_bar_sync(bar_id, NT);
#pragma unroll 8
    for (int m = 0; m < E; ++m) {
        const int pos = m * NT + tid;
        if (pos < n) {
            const uint32_t km = load_key(pos);
            if (((km - kmin) & pmask) == prefix) {
                const int slot = atomicAdd(&sc.misc[0], 1);
                if (slot < 64) sc.g64[slot] = comp_key(km, load_id(pos));
            }
        }
    }
    named_bar_sync(bar_id, NT);
    if (warp == 0) {
        for (int i = in_bin + lane; i < 64; i += 32) sc.g64[i] = 0ull;
        warp_sort64_desc(sc.g64, lane);
        if (lane == 0) sc.tau = sc.g64[remaining - 1];
    }
    named_bar_sync(bar_id, NT);
    const uint64_t tau = sc.tau;
    named_bar_sync(bar_id, NT);  // sc.tau and the scratch may be rewritten by the caller
    return tau;
}

// Stable compaction: every list position p < n with keep(p) is emitted as
// emit(out_pos, key, index), out_pos counting kept positions in list order.
// Returns the count. All NT threads call it with the same arguments. The
// emit may write the list in place: keys and indices are read a group of
// rounds ahead of the writes (round m's outputs land below (m + 1) * NT).
template <int NT, int E, class LoadKey, class LoadId, class Keep, class Emit>
__device__ int comp_compact(int n, int tid, int bar_id, CompScratch<NT, E>& sc, LoadKey&& load_key,
                            LoadId&& load_id, Keep&& keep, Emit&& emit) {
    constexpr int NW = NT / 32;
    constexpr int NTB = E * NW;
    const int lane = tid & 31, warp = tid >> 5;
    uint32_t kmask = 0;
#pragma unroll 8
    for (int m = 0; m < E; ++m) {
        const int pos = m * NT + tid;
        if (pos < n && keep(pos)) kmask |= 1u << m;
    }
    int my_s = 0;
#pragma unroll
    for (int m = 0; m < E; ++m) {
        const uint32_t bs = __ballot_sync(0xffffffffu, (kmask >> m) & 1u);
        if (lane == m) my_s = __popc(bs);
    }
    if (lane < E) sc.tbl[lane * NW + warp] = my_s;
    named_bar_sync(bar_id, NT);
    // exclusive scan of the (round, warp) table in list order
    static_assert(NTB <= NT, "one table entry per thread");
    const int ts = tid < NTB ? sc.tbl[tid] : 0;
    int ex, ex_b, tot, tot_b;
    block_scan2<NT>(ts, 0, ex, ex_b, tot, tot_b, sc.scan_tmp, tid, bar_id);
    if (tid < NTB) sc.tbl[tid] = ex;
    constexpr int GR = 4;
    uint32_t kb[GR];
    int32_t idb[GR];
    auto read_group = [&](int g) {
#pragma unroll
        for (int u = 0; u < GR; ++u) {
            const int m = g * GR + u;
            kb[u] = 0u;
            idb[u] = 0;
            if (m < E && ((kmask >> m) & 1u)) {
                kb[u] = load_key(m * NT + tid);
                idb[u] = load_id(m * NT + tid);
            }
        }
    };
    read_group(0);
    named_bar_sync(bar_id, NT);  // table published; group 0 read
    const uint32_t lt = lanemask_lt();
#pragma unroll
    for (int g = 0; g < (E + GR - 1) / GR; ++g) {
#pragma unroll
        for (int u = 0; u < GR; ++u) {
            const int m = g * GR + u;
            if (m < E) {
                const bool kp = (kmask >> m) & 1u;
                const uint32_t bs = __ballot_sync(0xffffffffu, kp);
                if (kp) emit(sc.tbl[m * NW + warp] + __popc(bs & lt), kb[u], idb[u]);
            }
        }
        read_group(g + 1);
        named_bar_sync(bar_id, NT);
    }
    return tot;
}

// Grouped stable emit: every list position p < n with keep(p) is emitted as
// emit(out_pos, p), ordered by group(p) in [0, 4) first and list order
// within a group. Returns the count. All NT threads call it with the same
// arguments; the list is only read.
template <int NT, int E, class Keep, class Group, class Emit>
__device__ int comp_emit_grouped(int n, int tid, int bar_id, CompScratch<NT, E>& sc, Keep&& keep, Group&& group,
                                 Emit&& emit) {
    constexpr int NW = NT / 32;
    constexpr int NTB = CompScratch<NT, E>::NTBL;
    const int lane = tid & 31, warp = tid >> 5;
    // bin of round m: its group (0..3), or -1 when the position is not kept;
    // two bits per round (group + 1 in 0..4 needs three: kept mask apart)
    uint32_t kmask = 0, gbits0 = 0, gbits1 = 0;
#pragma unroll 8
    for (int m = 0; m < E; ++m) {
        const int pos = m * NT + tid;
        if (pos < n && keep(pos)) {
            kmask |= 1u << m;
            const int g = group(pos);
            gbits0 |= static_cast<uint32_t>(g & 1) << m;
            gbits1 |= static_cast<uint32_t>((g >> 1) & 1) << m;
        }
    }
    auto bin_of = [&](int m) {
        return ((kmask >> m) & 1u) ? static_cast<int>(((gbits0 >> m) & 1u) | (((gbits1 >> m) & 1u) << 1)) : -1;
    };
    for (int i = tid; i < NTB; i += NT) sc.tbl[i] = 0;
    named_bar_sync(bar_id, NT);
    // per (group, round, warp): one ballot per group; lane g writes group g's count
#pragma unroll
    for (int m = 0; m < E; ++m) {
        const int b = bin_of(m);
        int mine = 0;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            const int c = __popc(__ballot_sync(0xffffffffu, b == g));
            if (lane == g) mine = c;
        }
        if (lane < 4) sc.tbl[(lane * E + m) * NW + warp] = mine;
    }
    named_bar_sync(bar_id, NT);
    // exclusive scan over the (group, round, warp) table: each thread scans a
    // run of consecutive entries, then a block scan of the run totals
    constexpr int RUN = (NTB + NT - 1) / NT;
    int run_vals[RUN];
    int run_sum = 0;
#pragma unroll
    for (int i = 0; i < RUN; ++i) {
        const int e = tid * RUN + i;
        run_vals[i] = e < NTB ? sc.tbl[e] : 0;
        run_sum += run_vals[i];
    }
    int ex, ex_b, tot, tot_b;
    block_scan2<NT>(run_sum, 0, ex, ex_b, tot, tot_b, sc.scan_tmp, tid, bar_id);
#pragma unroll
    for (int i = 0; i < RUN; ++i) {
        const int e = tid * RUN + i;
        if (e < NTB) sc.tbl[e] = ex;
        ex += run_vals[i];
    }
    named_bar_sync(bar_id, NT);
    const uint32_t lt = lanemask_lt();
#pragma unroll 4
    for (int m = 0; m < E; ++m) {
        const int b = bin_of(m);
        uint32_t peers = 0;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            const uint32_t bg = __ballot_sync(0xffffffffu, b == g);
            if (b == g) peers = bg;
        }
        if (b >= 0) emit(sc.tbl[(b * E + m) * NW + warp] + __popc(peers & lt), m * NT + tid);
    }
    named_bar_sync(bar_id, NT);  // the table may be reused
    return tot;
}

}  // namespace ic
