// C ABI of the B200 DSA / IndexCache hot path (declared in include/indexcache.h).
//
// Host responsibilities only: argument validation, kernel selection among the
// compiled shapes, TMA tensor-map encoding, launch geometry, workspace
// carving, and the IndexCache layer loop (IndexCache paper, Figure 2
// caption: one conditional branch per layer around the indexer, one index
// buffer overwritten by each Full layer). All arithmetic runs in the kernels
// of indexer.cuh and attention.cuh.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <limits>
#include <string>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "../../include/indexcache.h"
#include "attention.cuh"
#include "attention_pair.cuh"
#include "common.cuh"
#include "indexer.cuh"
#include "indexer_decode.cuh"
#include "distill.cuh"
#include "distill_tc.cuh"
#include "overlap.cuh"

namespace {

using ic::ceil_div;

thread_local char g_last_error[256] = "";

// Record a failed CUDA call (clearing the runtime's last-error slot) and map
// it to IC_ERR_CUDA.
ic_status cuda_fail(const char* what, cudaError_t e) {
    (void)cudaGetLastError();
    std::snprintf(g_last_error, sizeof g_last_error, "%s: %s", what, cudaGetErrorString(e));
    return IC_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Driver entry point for TMA descriptors (resolved at run time so the library
// loads on machines without a GPU driver).
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = []() -> EncodeTiledFn {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<EncodeTiledFn>(ptr);
    }();
    return fn;
}

// 2-D row-major tensor [rows, cols] with 128-byte swizzled boxes.
bool make_tmap(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int elem_bytes, uint64_t cols,
               uint64_t rows, uint32_t box_cols, uint32_t box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * static_cast<uint64_t>(elem_bytes)};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return enc(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct DeviceInfo {
    int sms = 0;
};

DeviceInfo device_info() {
    int dev = 0;
    DeviceInfo d;
    if (cudaGetDevice(&dev) != cudaSuccess) return d;
    cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
    return d;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Launch with an optional programmatic dependency on the previous kernel in
// the stream (it may still be finishing when this one starts; the kernels
// wait with griddep_wait before touching what it wrote). Only used when that
// previous kernel is one of this library's: a caller's kernel may write what
// a kernel reads before its wait.
cudaError_t launch(const void* kernel, dim3 grid, dim3 block, size_t smem, cudaStream_t stream, void** args,
                   bool pdl) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
#ifdef IC_NO_PDL
    cfg.numAttrs = 0;
    (void)pdl;
#else
    cfg.numAttrs = pdl ? 1 : 0;
#endif
    return cudaLaunchKernelExC(&cfg, kernel, args);
}
bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

// A kernel that rebalances registers with setmaxnreg must have been launched
// with at least `regs` registers per thread, or its warpgroups would wait for
// registers forever. The compiled count is checked once per kernel.
ic_status check_register_pool(const void* kernel, int regs) {
    static std::mutex mu;
    static std::vector<std::pair<const void*, int>> seen;
    std::lock_guard<std::mutex> lock(mu);
    for (auto& kv : seen)
        if (kv.first == kernel) return kv.second >= regs ? IC_OK : IC_ERR_UNSUPPORTED;
    cudaFuncAttributes attr;
    const cudaError_t e = cudaFuncGetAttributes(&attr, kernel);
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        return IC_ERR_CUDA;
    }
    seen.emplace_back(kernel, attr.numRegs);
    return attr.numRegs >= regs ? IC_OK : IC_ERR_UNSUPPORTED;
}

inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ---------------------------------------------------------------------------
// Indexer: compiled shapes
// ---------------------------------------------------------------------------
//            H_I  G   d_I  FP8    STAGES E (capacity = 128 E per query)
using IdxBf16H64 = ic::IdxCfg<64, 4, 128, false, 2, 22>;
using IdxFp8H64 = ic::IdxCfg<64, 4, 128, true, 3, 32>;
using IdxBf16H64G1 = ic::IdxCfg<64, 1, 128, false, 4, 32>;
using IdxFp8H64G1 = ic::IdxCfg<64, 1, 128, true, 4, 32>;
using IdxBf16H4 = ic::IdxCfg<4, 64, 64, false, 3, 2>;
// decode-style score rows (one query per sequence)
using IdxDecFp8 = ic::IdxDecCfg<128, true, 6>;
using IdxDecBf16 = ic::IdxDecCfg<128, false, 5>;

struct IdxPlan {
    int G = 0, C = 0, smem = 0, threads = 0, regs = 0;
    int step_keys = 0;  // keys one append step can add to a candidate list
    const void* kernel = nullptr;
    // decode-style score-row kernel (null where the shape has none)
    const void* dec_kernel = nullptr;
    int dec_smem = 0, dec_threads = 0, dec_regs = 0;
};

template <class Cfg>
void set_dec_plan(IdxPlan* pl) {
    pl->dec_kernel = reinterpret_cast<const void*>(&ic::indexer_decode_scores_kernel<Cfg>);
    pl->dec_smem = Cfg::SMEM_ALLOC;
    pl->dec_threads = Cfg::THREADS;
    pl->dec_regs = Cfg::REGS_LAUNCH;
}

template <class Cfg>
IdxPlan idx_plan() {
    IdxPlan pl;
    pl.G = Cfg::G;
    pl.C = Cfg::C;
    // room a list needs above topk: one append step (generic path); the FAST
    // path's cut must leave the list below its high-water mark (topk + 3 tiles)
    pl.step_keys = Cfg::FAST ? 3 * ic::IDX_BM : ic::IDX_BM * Cfg::PSTEP;
    pl.smem = Cfg::SMEM_ALLOC;
    pl.threads = Cfg::THREADS;
    pl.regs = Cfg::REGS_LAUNCH;
    pl.kernel = reinterpret_cast<const void*>(&ic::indexer_topk_kernel<Cfg>);
    return pl;
}

bool choose_idx_plan(int H_I, int d_I, ic_dtype qk, int n_q, IdxPlan* pl) {
    const bool single = n_q == 1;
    if (H_I == 64 && d_I == 128 && qk == IC_BF16) {
        *pl = single ? idx_plan<IdxBf16H64G1>() : idx_plan<IdxBf16H64>();
        if (single) set_dec_plan<IdxDecBf16>(pl);
        return true;
    }
    if (H_I == 64 && d_I == 128 && qk == IC_FP8_E4M3) {
        *pl = single ? idx_plan<IdxFp8H64G1>() : idx_plan<IdxFp8H64>();
        if (single) set_dec_plan<IdxDecFp8>(pl);
        return true;
    }
    if (H_I == 4 && d_I == 64 && qk == IC_BF16) {
        *pl = idx_plan<IdxBf16H4>();
        return true;
    }
    return false;
}

// The top-k plus the keys of one append step must fit a query's candidate list.
bool plan_supports_topk(const IdxPlan& pl, int topk) { return topk + pl.step_keys <= pl.C && topk <= 2048; }

constexpr int MERGE_E = 32;              // merge kernel: up to 256 * 32 candidates per row
constexpr int MERGE_MAX = 256 * MERGE_E;

int idx_splits(const IdxPlan& pl, int batch, int n_q, int n_k, int topk, int sms) {
    if (n_q != 1 || sms <= 0) return 1;
    int s = ceil_div(sms, std::max(batch, 1));
    s = std::min(s, MERGE_MAX / topk);
    s = std::min(s, std::max(1, n_k / (2 * topk)));
    s = std::min(s, 8);
    (void)pl;
    return std::max(s, 1);
}

struct IdxLayout {
    int splits = 1, chunk = 0;
    size_t off_key = 0, off_idx = 0, off_cnt = 0, bytes = 0;
    bool dense = false;  // decode-style score rows + per-row select
    int stride = 0;      // score-row stride (keys)
};

// allow_dense = false keeps decode-style calls on the split candidate lists,
// whose scratch does not grow with the number of visible keys.
IdxLayout idx_layout(const IdxPlan& pl, int batch, int n_q, int n_k, int topk, int sms, bool allow_dense = true) {
    IdxLayout L;
    if (allow_dense && n_q == 1 && pl.dec_kernel != nullptr && n_k >= 1 && n_k <= ic::TOPK_ROWS_MAX) {
        L.dense = true;
        L.stride = static_cast<int>(round_up(static_cast<size_t>(n_k), ic::IDX_BM));
        L.bytes = round_up(static_cast<size_t>(batch) * L.stride * 4, 256);
        return L;
    }
    L.splits = idx_splits(pl, batch, n_q, n_k, topk, sms);
    L.chunk = static_cast<int>(round_up(static_cast<size_t>(ceil_div(std::max(n_k, 1), L.splits)), ic::IDX_BM));
    if (L.splits > 1) {
        const size_t rows = static_cast<size_t>(batch) * n_q;
        const size_t n = rows * L.splits * topk;
        L.off_key = 0;
        L.off_idx = round_up(n * 4, 256);
        L.off_cnt = L.off_idx + round_up(n * 4, 256);
        L.bytes = L.off_cnt + round_up(rows * L.splits * 4, 256);
    }
    return L;
}

ic_status validate_indexer(const void* q_I, const float* q_scale, const void* w, ic_dtype w_dt, const void* k_I,
                           const float* k_scale, ic_dtype qk_dt, int batch, int n_q, int n_k, int q_pos0,
                           int H_I, int d_I, int topk, const int32_t* idx_out) {
    if (batch < 0 || n_q < 0 || n_k < 0 || q_pos0 < 0 || H_I <= 0 || d_I <= 0 || topk <= 0)
        return IC_ERR_INVALID_ARG;
    if (qk_dt != IC_BF16 && qk_dt != IC_FP8_E4M3) return IC_ERR_INVALID_ARG;
    if (w_dt != IC_BF16 && w_dt != IC_F32) return IC_ERR_INVALID_ARG;
    if (static_cast<int64_t>(q_pos0) + n_q > (int64_t{1} << 30)) return IC_ERR_INVALID_ARG;
    if (batch == 0 || n_q == 0) return IC_OK;
    if (!q_I || !w || !idx_out || (n_k > 0 && !k_I)) return IC_ERR_INVALID_ARG;
    if (qk_dt == IC_FP8_E4M3 && (!q_scale || (n_k > 0 && !k_scale))) return IC_ERR_INVALID_ARG;
    if (!aligned16(q_I) || (n_k > 0 && !aligned16(k_I))) return IC_ERR_INVALID_ARG;
    return IC_OK;
}

ic_status launch_indexer(const void* q_I, const float* q_scale, const void* w, ic_dtype w_dt, const void* k_I,
                         const float* k_scale, ic_dtype qk_dt, int batch, int n_q, int n_k, int q_pos0, int H_I,
                         int d_I, int topk, int32_t* idx_out, void* ws, size_t ws_bytes, cudaStream_t stream,
                         bool allow_dense = true, bool pdl = false) {
    ic_status st = validate_indexer(q_I, q_scale, w, w_dt, k_I, k_scale, qk_dt, batch, n_q, n_k, q_pos0, H_I,
                                    d_I, topk, idx_out);
    if (st != IC_OK) return st;
    if (batch == 0 || n_q == 0) return IC_OK;
    // the scratch holds 256-byte aligned sub-arrays read with vector loads
    if (ws != nullptr && !aligned256(ws)) return IC_ERR_WORKSPACE;
    IdxPlan pl;
    if (!choose_idx_plan(H_I, d_I, qk_dt, n_q, &pl)) return IC_ERR_UNSUPPORTED;
    if (!plan_supports_topk(pl, topk)) return IC_ERR_UNSUPPORTED;
    const DeviceInfo dev = device_info();
    if (dev.sms <= 0) return cuda_fail("device query", cudaErrorNoDevice);
    const IdxLayout L = idx_layout(pl, batch, n_q, n_k, topk, dev.sms, allow_dense);
    if (L.bytes > 0 && (ws == nullptr || ws_bytes < L.bytes)) return IC_ERR_WORKSPACE;

    const int esz = qk_dt == IC_FP8_E4M3 ? 1 : 2;
    const CUtensorMapDataType tdt = qk_dt == IC_FP8_E4M3 ? CU_TENSOR_MAP_DATA_TYPE_UINT8
                                                         : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const uint32_t atom_elems = 128 / esz;
    CUtensorMap tm_q, tm_k;
    const uint64_t q_rows = static_cast<uint64_t>(batch) * n_q * H_I;
    const uint64_t k_rows = std::max<uint64_t>(static_cast<uint64_t>(batch) * n_k, 1);
    if (!make_tmap(&tm_q, q_I, tdt, esz, d_I, q_rows, atom_elems, pl.G * H_I))
        return cuda_fail("q_I tensor map", cudaErrorInvalidValue);
    if (!make_tmap(&tm_k, n_k > 0 ? k_I : q_I, tdt, esz, d_I, n_k > 0 ? k_rows : q_rows, atom_elems, ic::IDX_BM))
        return cuda_fail("k_I tensor map", cudaErrorInvalidValue);

    if (L.dense) {
        // decode-style: score rows of the visible keys, then one exact select per row
        ic::IdxDecParams d;
        d.w = w;
        d.q_scale = q_scale;
        d.k_scale = k_scale;
        d.w_is_f32 = w_dt == IC_F32 ? 1 : 0;
        d.batch = batch;
        d.n_k = n_k;
        d.n_vis = std::min(q_pos0 + 1, n_k);
        d.n_chunks = ceil_div(ceil_div(d.n_vis, ic::IDX_BM), ic::IDX_DEC_CHUNK);
        d.n_work = batch * d.n_chunks;
        d.stride = L.stride;
        d.scores = static_cast<uint32_t*>(ws);
        if (check_register_pool(pl.dec_kernel, pl.dec_regs) != IC_OK)
            return cuda_fail("decode indexer register pool", cudaErrorInvalidConfiguration);
        cudaError_t e = cudaFuncSetAttribute(pl.dec_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, pl.dec_smem);
        if (e != cudaSuccess) return cuda_fail("decode indexer smem attribute", e);
        const int grid = std::max(1, std::min(d.n_work, dev.sms));
        void* args[] = {&tm_q, &tm_k, &d};
        e = launch(pl.dec_kernel, dim3(grid), dim3(pl.dec_threads), pl.dec_smem, stream, args, pdl);
        if (e != cudaSuccess) return cuda_fail("decode indexer launch", e);
        const uint32_t* sc_ptr = d.scores;
        int stride = d.stride, n_vis = d.n_vis, kk = topk;
        void* rargs[] = {&sc_ptr, &stride, &n_vis, &kk, &idx_out};
        e = launch(reinterpret_cast<const void*>(&ic::topk_rows_kernel), dim3(batch * ic::TOPK_ROWS_CL),
                   dim3(ic::TOPK_ROWS_NT), 0, stream, rargs, true);
        if (e != cudaSuccess) return cuda_fail("top-k rows launch", e);
        return IC_OK;
    }

    ic::IdxParams p;
    p.w = w;
    p.q_scale = q_scale;
    p.k_scale = k_scale;
    p.w_is_f32 = w_dt == IC_F32 ? 1 : 0;
    p.batch = batch;
    p.n_q = n_q;
    p.n_k = n_k;
    p.q_pos0 = q_pos0;
    p.topk = topk;
    p.n_groups = ceil_div(n_q, pl.G);
    p.n_splits = L.splits;
    p.chunk = L.chunk;
    p.n_work = p.n_groups * batch * L.splits;
    p.idx_out = idx_out;
    uint8_t* wsb = static_cast<uint8_t*>(ws);
    p.cand_key = L.splits > 1 ? reinterpret_cast<uint32_t*>(wsb + L.off_key) : nullptr;
    p.cand_idx = L.splits > 1 ? reinterpret_cast<int32_t*>(wsb + L.off_idx) : nullptr;
    p.cand_cnt = L.splits > 1 ? reinterpret_cast<int32_t*>(wsb + L.off_cnt) : nullptr;

    if (check_register_pool(pl.kernel, pl.regs) != IC_OK)
        return cuda_fail("indexer register pool", cudaErrorInvalidConfiguration);
    cudaError_t e = cudaFuncSetAttribute(pl.kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, pl.smem);
    if (e != cudaSuccess) return cuda_fail("indexer smem attribute", e);
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, pl.kernel, pl.threads, pl.smem);
    if (e != cudaSuccess) return cuda_fail("indexer occupancy", e);
    if (per_sm < 1) return cuda_fail("indexer occupancy", cudaErrorInvalidConfiguration);
    const int grid = std::max(1, std::min(p.n_work, dev.sms * per_sm));
    void* args[] = {&tm_q, &tm_k, &p};
    e = launch(pl.kernel, dim3(grid), dim3(pl.threads), pl.smem, stream, args, pdl);
    if (e != cudaSuccess) return cuda_fail("indexer launch", e);
    if (L.splits > 1) {
        constexpr int merge_smem = MERGE_MAX * 8;
        e = cudaFuncSetAttribute(&ic::topk_merge_kernel<MERGE_E>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 merge_smem);
        if (e != cudaSuccess) return cuda_fail("top-k merge smem attribute", e);
        const uint32_t* ckp = p.cand_key;
        const int32_t* cip = p.cand_idx;
        const int32_t* ccp = p.cand_cnt;
        int splits = L.splits, kk = topk;
        void* margs[] = {&ckp, &cip, &ccp, &splits, &kk, &idx_out};
        e = launch(reinterpret_cast<const void*>(&ic::topk_merge_kernel<MERGE_E>), dim3(batch * n_q), dim3(256),
                   merge_smem, stream, margs, true);
        if (e != cudaSuccess) return cuda_fail("top-k merge launch", e);
    }
    return IC_OK;
}

// ---------------------------------------------------------------------------
// Attention: compiled shapes
// ---------------------------------------------------------------------------
using Attn576 = ic::AttnCfg<576, 512>;
using Attn64 = ic::AttnCfg<64, 64>;

struct AttnPlan {
    int smem = 0, threads = 0, dv = 0, regs = 0;
    const void* kernel = nullptr;
    void (*combine)(const float*, const float*, int, int, __nv_bfloat16*) = nullptr;
};

// The 576 / 512 latent shape forms the scores of two 64-key tiles per MMA
// chain (attention_pair.cuh); IC_ATTN_PAIR=0 selects the one-tile kernel.
#ifndef IC_ATTN_PAIR
#define IC_ATTN_PAIR 1
#endif

template <class Cfg, bool PAIR = false>
AttnPlan attn_plan() {
    AttnPlan pl;
    pl.smem = Cfg::SMEM_ALLOC;
    pl.threads = Cfg::THREADS;
    pl.dv = Cfg::DV;
    pl.regs = 65536 / Cfg::THREADS;
    if constexpr (PAIR)
        pl.kernel = reinterpret_cast<const void*>(&ic::sparse_attn_pair_kernel<Cfg>);
    else
        pl.kernel = reinterpret_cast<const void*>(&ic::sparse_attn_kernel<Cfg>);
    pl.combine = &ic::attn_combine_kernel<Cfg::DV>;
    return pl;
}

bool choose_attn_plan(int d_qk, int d_v, AttnPlan* pl) {
    if (d_qk == 576 && d_v == 512) {
        *pl = attn_plan<Attn576, IC_ATTN_PAIR != 0>();
        return true;
    }
    if (d_qk == 64 && d_v == 64) {
        *pl = attn_plan<Attn64>();
        return true;
    }
    return false;
}

#ifndef IC_ATTN_SPLIT_WAVES
#define IC_ATTN_SPLIT_WAVES 1
#endif

int attn_splits(int rows, int topk, int sms) {
    if (rows <= 0 || sms <= 0 || rows >= sms) return 1;
    int s = IC_ATTN_SPLIT_WAVES * sms / rows;  // rounds of work items per CTA
    s = std::min(s, std::max(1, ceil_div(topk, 256)));
    s = std::min(s, 8);
    return std::max(s, 1);
}

size_t attn_ws_bytes(int rows, int splits, int H, int d_v) {
    if (splits <= 1) return 0;
    const size_t slots = static_cast<size_t>(rows) * splits;
    return round_up(slots * H * d_v * 4, 256) + round_up(slots * 128 * 4, 256);
}

ic_status launch_attn(const void* q, const void* kv, const int32_t* idx, int batch, int n_q, int n_k, int H, int d_qk,
                      int d_v, int topk, float sm_scale, void* out, void* ws, size_t ws_bytes,
                      cudaStream_t stream, bool pdl = false) {
    if (batch < 0 || n_q < 0 || n_k < 0 || H <= 0 || d_qk <= 0 || d_v <= 0 || topk <= 0) return IC_ERR_INVALID_ARG;
    if (batch == 0 || n_q == 0) return IC_OK;
    if (!q || !idx || !out || (n_k > 0 && !kv)) return IC_ERR_INVALID_ARG;
    if (!aligned16(q) || (n_k > 0 && !aligned16(kv))) return IC_ERR_INVALID_ARG;
    // the split partials are 256-byte aligned sub-arrays read with vector loads
    if (ws != nullptr && !aligned256(ws)) return IC_ERR_WORKSPACE;
    AttnPlan pl;
    if (!choose_attn_plan(d_qk, d_v, &pl)) return IC_ERR_UNSUPPORTED;
    if (H > 64 || topk > ic::AttnCfg<64, 64>::MAX_TOPK) return IC_ERR_UNSUPPORTED;
    const DeviceInfo dev = device_info();
    if (dev.sms <= 0) return cuda_fail("device query", cudaErrorNoDevice);
    const int rows = batch * n_q;
    const int splits = attn_splits(rows, topk, dev.sms);
    const size_t need = attn_ws_bytes(rows, splits, H, d_v);
    if (need > 0 && (ws == nullptr || ws_bytes < need)) return IC_ERR_WORKSPACE;

    CUtensorMap tm_q, tm_kv;
    if (!make_tmap(&tm_q, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d_qk, static_cast<uint64_t>(rows) * H, 64, H))
        return cuda_fail("q tensor map", cudaErrorInvalidValue);
    // row-gather map over the latent KV: one-row boxes of 64 columns
    if (!make_tmap(&tm_kv, n_k > 0 ? kv : q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, d_qk,
                   n_k > 0 ? static_cast<uint64_t>(batch) * n_k : static_cast<uint64_t>(rows) * H, 64, 1))
        return cuda_fail("kv tensor map", cudaErrorInvalidValue);
    ic::AttnParams p;
    p.kv = static_cast<const __nv_bfloat16*>(n_k > 0 ? kv : q);
    p.idx = idx;
    p.out = static_cast<__nv_bfloat16*>(out);
    uint8_t* wsb = static_cast<uint8_t*>(ws);
    const size_t slots = static_cast<size_t>(rows) * splits;
    p.o_part = splits > 1 ? reinterpret_cast<float*>(wsb) : nullptr;
    p.ml_part = splits > 1 ? reinterpret_cast<float*>(wsb + round_up(slots * H * d_v * 4, 256)) : nullptr;
    p.batch = batch;
    p.n_q = n_q;
    p.n_k = n_k;
    p.H = H;
    p.topk = topk;
    p.sm_scale_log2 = sm_scale * 1.4426950408889634f;
    p.n_splits = splits;
    p.n_work = rows * splits;
    if (check_register_pool(pl.kernel, pl.regs) != IC_OK)
        return cuda_fail("attention register pool", cudaErrorInvalidConfiguration);
    cudaError_t e = cudaFuncSetAttribute(pl.kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, pl.smem);
    if (e != cudaSuccess) return cuda_fail("attention smem attribute", e);
    const int grid = std::max(1, std::min(p.n_work, dev.sms));
    void* args[] = {&tm_q, &tm_kv, &p};
    e = launch(pl.kernel, dim3(grid), dim3(pl.threads), pl.smem, stream, args, pdl);
    if (e != cudaSuccess) return cuda_fail("attention launch", e);
    if (splits > 1) {
        int sp = splits, hh = H;
        void* cargs[] = {&p.o_part, &p.ml_part, &sp, &hh, &p.out};
        e = launch(reinterpret_cast<const void*>(pl.combine), dim3(rows * H), dim3(128), 0, stream, cargs, true);
        if (e != cudaSuccess) return cuda_fail("attention combine launch", e);
    }
    return IC_OK;
}

__global__ void expire_wait_kernel(long long timeout_ns) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        ic::mbar_init(ic::smem_u32(&bar), 1);
        abort_flag = 0;
        ic::fence_mbar_init();
        // nothing ever arrives on this barrier: the wait must expire
        ic::mbar_wait(ic::smem_u32(&bar), 0, &abort_flag, static_cast<uint64_t>(timeout_ns));
    }
}

}  // namespace

// ---------------------------------------------------------------------------
// Scratch for ic_indexer_topk_noalloc: a fixed device array owned by the
// library, so that entry point never allocates. Every device that loads this
// library holds it until the process exits.
// ---------------------------------------------------------------------------
#define IC_NOALLOC_SCRATCH_BYTES (8u << 20)
static __device__ __align__(256) uint8_t g_noalloc_scratch[IC_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device. The name is a
// host-side stand-in in host code; the real address comes from
// cudaGetSymbolAddress, resolved once per device with that device current.
ic_status noalloc_scratch(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail("no-alloc scratch: current device", e);
    if (dev < 0 || dev >= kMaxDevices) return cuda_fail("no-alloc scratch: device ordinal", cudaErrorInvalidDevice);
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (g_noalloc_ptr[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail("no-alloc scratch: cudaGetSymbolAddress", e);
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return IC_OK;
}


template <int DQK, int HI>
ic_status launch_distill(const ic::DistillParams& p, int rows, cudaStream_t stream) {
    const size_t smem = ic::distill_smem_bytes(DQK, HI, p.d_I, p.topk);
    cudaError_t e = cudaFuncSetAttribute(ic::distill_target_kernel<DQK, HI>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return cuda_fail("distill smem attribute", e);
    ic::distill_target_kernel<DQK, HI><<<rows, ic::DISTILL_THREADS, smem, stream>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail("distill launch", e);
    return IC_OK;
}

// The model's shapes run on the tensor cores; other shapes on the CUDA cores.
bool distill_on_tensor_cores(int H, int d_qk, int H_I, int d_I) {
    return H == 64 && d_qk == 576 && H_I == 64 && d_I == 128;
}

// Grid of the tensor-core kernel (persistent CTAs, one query row at a time)
// and its workspace: the spilled logits of up to SPILL_TILES tiles per CTA
// (only rows of more than RESIDENT tiles, i.e. topk > 1024, spill).
using DistTcAny = ic::DistTcCfg<576, true>;
static_assert(DistTcAny::SPILL_BYTES_PER_CTA == ic::DistTcCfg<576, false>::SPILL_BYTES_PER_CTA, "spill size");
int distill_tc_grid(int rows, int sms) { return std::max(1, std::min(rows, sms)); }
size_t distill_tc_ws_bytes(int rows, int topk, int sms) {
    if (topk <= DistTcAny::RESIDENT * DistTcAny::BM) return 0;
    return DistTcAny::SPILL_BYTES_PER_CTA * static_cast<size_t>(distill_tc_grid(rows, sms));
}

template <class Cfg>
ic_status launch_distill_tc(const ic::DistillParams& p, int sms, cudaStream_t stream) {
    cudaError_t e = cudaFuncSetAttribute(ic::distill_tc_kernel<Cfg>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         Cfg::SMEM_ALLOC);
    if (e != cudaSuccess) return cuda_fail("distill (tensor cores) smem attribute", e);
    ic::distill_tc_kernel<Cfg><<<distill_tc_grid(p.rows, sms), Cfg::THREADS, Cfg::SMEM_ALLOC, stream>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail("distill (tensor cores) launch", e);
    return IC_OK;
}

}  // namespace

extern "C" {

// ---------------------------------------------------------------------------
// Pattern tools
// ---------------------------------------------------------------------------
ic_status ic_topk_overlap(const int32_t* idx_a, const int32_t* idx_b, int rows, int topk, int n_k, int32_t* counts_out,
                          void* stream) {
    if (rows < 0 || topk <= 0 || n_k < 0) return IC_ERR_INVALID_ARG;
    if (rows == 0) return IC_OK;
    if (!idx_a || !idx_b || !counts_out) return IC_ERR_INVALID_ARG;
    const size_t bits_bytes = static_cast<size_t>((std::max(n_k, 1) + 31) / 32) * 4;
    if (bits_bytes > 225 * 1024) return IC_ERR_UNSUPPORTED;
    const DeviceInfo dev = device_info();
    if (dev.sms <= 0) return cuda_fail("device query", cudaErrorNoDevice);
    cudaError_t e = cudaFuncSetAttribute(&ic::topk_overlap_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(bits_bytes));
    if (e != cudaSuccess) return cuda_fail("overlap smem attribute", e);
    const int grid = std::max(1, std::min(rows, 2 * dev.sms));
    ic::topk_overlap_kernel<<<grid, ic::OVERLAP_THREADS, bits_bytes, static_cast<cudaStream_t>(stream)>>>(
        idx_a, idx_b, rows, topk, n_k, counts_out);
    e = cudaGetLastError();
    return e == cudaSuccess ? IC_OK : cuda_fail("overlap launch", e);
}

ic_status ic_overlap_matrix_workspace_size(int n_layers, size_t* bytes_out) {
    if (!bytes_out || n_layers < 1 || n_layers > ic::OVERLAP_MAX_LAYERS) return IC_ERR_INVALID_ARG;
    *bytes_out = round_up(static_cast<size_t>(n_layers) * n_layers * sizeof(unsigned long long), 256);
    return IC_OK;
}

ic_status ic_overlap_matrix(const int32_t* const* idx_layers, int n_layers, int rows, int topk, int n_k,
                            void* workspace, size_t workspace_bytes, double* ratio_out, void* stream) {
    if (!idx_layers || !ratio_out || n_layers < 1 || rows < 0 || topk <= 0 || n_k < 0) return IC_ERR_INVALID_ARG;
    if (n_layers > ic::OVERLAP_MAX_LAYERS) return IC_ERR_UNSUPPORTED;
    for (int l = 0; l < n_layers; ++l)
        if (!idx_layers[l]) return IC_ERR_INVALID_ARG;
    const size_t bits_bytes = static_cast<size_t>((std::max(n_k, 1) + 31) / 32) * 4;
    if (bits_bytes > 224 * 1024) return IC_ERR_UNSUPPORTED;
    const size_t need = static_cast<size_t>(n_layers) * n_layers * sizeof(unsigned long long);
    if (!workspace || workspace_bytes < need) return IC_ERR_WORKSPACE;
    const DeviceInfo dev = device_info();
    if (dev.sms <= 0) return cuda_fail("device query", cudaErrorNoDevice);
    const cudaStream_t cs = static_cast<cudaStream_t>(stream);
    unsigned long long* counts = static_cast<unsigned long long*>(workspace);
    cudaError_t e = cudaMemsetAsync(counts, 0, need, cs);
    if (e != cudaSuccess) return cuda_fail("overlap counts reset", e);
    if (rows > 0) {
        ic::OverlapLayers L{};
        for (int l = 0; l < n_layers; ++l) L.p[l] = idx_layers[l];
        e = cudaFuncSetAttribute(&ic::overlap_counts_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(bits_bytes));
        if (e != cudaSuccess) return cuda_fail("overlap smem attribute", e);
        const int grid = std::max(1, std::min(rows, dev.sms));
        for (int a = 0; a < n_layers; ++a) {
            ic::overlap_counts_kernel<<<grid, ic::OVERLAP_THREADS, bits_bytes, cs>>>(L, a, n_layers, rows, topk, n_k,
                                                                                   counts);
            e = cudaGetLastError();
            if (e != cudaSuccess) return cuda_fail("overlap counts launch", e);
        }
    }
    std::vector<unsigned long long> host(static_cast<size_t>(n_layers) * n_layers);
    e = cudaMemcpyAsync(host.data(), counts, need, cudaMemcpyDeviceToHost, cs);
    if (e != cudaSuccess) return cuda_fail("overlap counts copy", e);
    e = cudaStreamSynchronize(cs);
    if (e != cudaSuccess) return cuda_fail("overlap counts synchronize", e);
    // R[a][b] = overlap counts over layer a's valid entries (the diagonal)
    for (int a = 0; a < n_layers; ++a) {
        const double valid = static_cast<double>(host[static_cast<size_t>(a) * n_layers + a]);
        for (int b = 0; b < n_layers; ++b) {
            const size_t i = static_cast<size_t>(a) * n_layers + b;
            ratio_out[i] = a == b ? 1.0 : static_cast<double>(host[i]) / std::max(valid, 1.0);
        }
    }
    return IC_OK;
}

ic_status ic_pattern_score(const double* overlap, int n_layers, const char* pattern, double* score_out) {
    if (!overlap || !pattern || !score_out || n_layers < 1) return IC_ERR_INVALID_ARG;
    if (std::strlen(pattern) != static_cast<size_t>(n_layers) || pattern[0] != 'F') return IC_ERR_BAD_PATTERN;
    double s = 0.0;
    int src = 0;
    for (int l = 0; l < n_layers; ++l) {
        if (pattern[l] == 'F') src = l;
        else if (pattern[l] != 'S') return IC_ERR_BAD_PATTERN;
        s += overlap[static_cast<size_t>(l) * n_layers + src];
    }
    *score_out = s;
    return IC_OK;
}

ic_status ic_search_pattern(const double* overlap, int n_layers, int n_full, char* pattern_out, double* score_out) {
    if (!overlap || !pattern_out || n_layers <= 0 || n_full < 1 || n_full > n_layers) return IC_ERR_INVALID_ARG;
    const int n = n_layers;
    for (int i = 0; i < n * n; ++i)
        if (!std::isfinite(overlap[i])) return IC_ERR_INVALID_ARG;
    // seg[i][j]: layers i..j-1 all served by Full layer i
    std::vector<double> seg(static_cast<size_t>(n) * (n + 1), 0.0);
    for (int i = 0; i < n; ++i) {
        double acc = 0.0;
        for (int j = i + 1; j <= n; ++j) {
            acc += overlap[static_cast<size_t>(j - 1) * n + i];
            seg[static_cast<size_t>(i) * (n + 1) + j] = acc;
        }
    }
    // best[c][j]: layers 0..j-1 covered by c segments, the first starting at 0
    const double NEG = -std::numeric_limits<double>::infinity();
    std::vector<double> best(static_cast<size_t>(n_full + 1) * (n + 1), NEG);
    std::vector<int> from(static_cast<size_t>(n_full + 1) * (n + 1), -1);
    auto B = [&](int c, int j) -> double& { return best[static_cast<size_t>(c) * (n + 1) + j]; };
    auto F = [&](int c, int j) -> int& { return from[static_cast<size_t>(c) * (n + 1) + j]; };
    for (int j = 1; j <= n; ++j) {
        B(1, j) = seg[j];
        F(1, j) = 0;
    }
    for (int c = 2; c <= n_full; ++c) {
        for (int j = c; j <= n; ++j) {
            for (int i = c - 1; i < j; ++i) {  // last segment starts at Full layer i
                if (B(c - 1, i) == NEG) continue;
                const double v = B(c - 1, i) + seg[static_cast<size_t>(i) * (n + 1) + j];
                if (v > B(c, j)) {
                    B(c, j) = v;
                    F(c, j) = i;
                }
            }
        }
    }
    for (int l = 0; l < n; ++l) pattern_out[l] = 'S';
    pattern_out[n] = 0;
    int j = n;
    for (int c = n_full; c >= 1; --c) {
        const int i = F(c, j);
        if (i < 0) return IC_ERR_INVALID_ARG;
        pattern_out[i] = 'F';
        j = i;
    }
    if (score_out) *score_out = B(n_full, n);
    return IC_OK;
}

ic_status ic_greedy_pattern(int n_layers, int n_full, ic_pattern_objective objective, void* ctx, char* pattern_out,
                            double* value_out) {
    if (!objective || !pattern_out || n_layers <= 0 || n_full < 1 || n_full > n_layers) return IC_ERR_INVALID_ARG;
    std::string pat(static_cast<size_t>(n_layers), 'F');
    double value = objective(pat.c_str(), ctx);
    if (!std::isfinite(value)) return IC_ERR_INVALID_ARG;
    for (int full = n_layers; full > n_full; --full) {
        int best_l = -1;
        double best_v = std::numeric_limits<double>::infinity();
        for (int l = 1; l < n_layers; ++l) {
            if (pat[l] != 'F') continue;
            pat[l] = 'S';
            const double v = objective(pat.c_str(), ctx);
            pat[l] = 'F';
            if (!std::isfinite(v)) return IC_ERR_INVALID_ARG;
            if (v < best_v) {
                best_v = v;
                best_l = l;
            }
        }
        if (best_l < 0) return IC_ERR_INVALID_ARG;
        pat[best_l] = 'S';
        value = best_v;
    }
    std::memcpy(pattern_out, pat.c_str(), static_cast<size_t>(n_layers) + 1);
    if (value_out) *value_out = value;
    return IC_OK;
}

const char* ic_status_string(ic_status s) {
    switch (s) {
        case IC_OK: return "IC_OK";
        case IC_ERR_INVALID_ARG: return "IC_ERR_INVALID_ARG";
        case IC_ERR_BAD_PATTERN: return "IC_ERR_BAD_PATTERN";
        case IC_ERR_UNSUPPORTED: return "IC_ERR_UNSUPPORTED";
        case IC_ERR_CUDA: return "IC_ERR_CUDA";
        case IC_ERR_TIMEOUT: return "IC_ERR_TIMEOUT";
        case IC_ERR_WORKSPACE: return "IC_ERR_WORKSPACE";
        case IC_ERR_INTERNAL: return "IC_ERR_INTERNAL";
    }
    return "IC_ERR_UNKNOWN";
}

int ic_version(void) { return (1 << 16) | 0; }

ic_status ic_resolve_pattern(int n_layers, int index_topk_freq, const char* index_topk_pattern,
                             uint8_t* is_full_out, int32_t* src_layer_out) {
    if (n_layers < 1 || index_topk_freq < 0 || !is_full_out || !src_layer_out) return IC_ERR_INVALID_ARG;
    if (index_topk_pattern != nullptr && index_topk_freq != 0) return IC_ERR_INVALID_ARG;
    if (index_topk_pattern != nullptr) {
        if (std::strlen(index_topk_pattern) != static_cast<size_t>(n_layers)) return IC_ERR_BAD_PATTERN;
        for (int l = 0; l < n_layers; ++l)
            if (index_topk_pattern[l] != 'F' && index_topk_pattern[l] != 'S') return IC_ERR_BAD_PATTERN;
        if (index_topk_pattern[0] != 'F') return IC_ERR_BAD_PATTERN;
    }
    int last = -1;
    for (int l = 0; l < n_layers; ++l) {
        bool full;
        if (index_topk_pattern != nullptr)
            full = index_topk_pattern[l] == 'F';
        else if (index_topk_freq >= 1)
            full = (l % index_topk_freq) == 0;
        else
            full = true;
        is_full_out[l] = full ? 1 : 0;
        if (full) last = l;
        src_layer_out[l] = last;
    }
    return IC_OK;
}

ic_status ic_indexer_workspace_size(int batch, int n_q, int n_k, int H_I, int d_I, int topk, ic_dtype qk_dtype,
                                    size_t* bytes_out) {
    if (!bytes_out || batch < 0 || n_q < 0 || n_k < 0 || topk <= 0) return IC_ERR_INVALID_ARG;
    *bytes_out = 0;
    if (batch == 0 || n_q == 0) return IC_OK;
    IdxPlan pl;
    if (!choose_idx_plan(H_I, d_I, qk_dtype, n_q, &pl) || !plan_supports_topk(pl, topk)) return IC_ERR_UNSUPPORTED;
    const DeviceInfo dev = device_info();
    if (dev.sms <= 0) return cuda_fail("device query", cudaErrorNoDevice);
    *bytes_out = idx_layout(pl, batch, n_q, n_k, topk, dev.sms).bytes;
    return IC_OK;
}

ic_status ic_indexer_topk(const void* q_I, const float* q_scale, const void* w, ic_dtype w_dtype, const void* k_I,
                          const float* k_scale, ic_dtype qk_dtype, int batch, int n_q, int n_k, int q_pos0, int H_I,
                          int d_I, int topk, int32_t* idx_out, void* workspace, size_t workspace_bytes,
                          void* stream) {
    return launch_indexer(q_I, q_scale, w, w_dtype, k_I, k_scale, qk_dtype, batch, n_q, n_k, q_pos0, H_I, d_I, topk,
                          idx_out, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

ic_status ic_sparse_attn_workspace_size(int batch, int n_q, int H, int d_v, int topk, size_t* bytes_out) {
    if (!bytes_out || batch < 0 || n_q < 0 || H <= 0 || d_v <= 0 || topk <= 0) return IC_ERR_INVALID_ARG;
    const DeviceInfo dev = device_info();
    if (dev.sms <= 0) return cuda_fail("device query", cudaErrorNoDevice);
    const int rows = batch * n_q;
    *bytes_out = attn_ws_bytes(rows, attn_splits(rows, topk, dev.sms), H, d_v);
    return IC_OK;
}

ic_status ic_sparse_attn(const void* q, const void* kv, const int32_t* idx, int batch, int n_q, int n_k, int H,
                         int d_qk, int d_v, int topk, float sm_scale, void* out, void* workspace,
                         size_t workspace_bytes, void* stream) {
    return launch_attn(q, kv, idx, batch, n_q, n_k, H, d_qk, d_v, topk, sm_scale, out, workspace, workspace_bytes,
                       static_cast<cudaStream_t>(stream));
}

ic_status ic_layer_stack_workspace_size(const ic_stack_shape* s, size_t* bytes_out) {
    if (!s || !bytes_out) return IC_ERR_INVALID_ARG;
    size_t a = 0, b = 0;
    ic_status st = ic_indexer_workspace_size(s->batch, s->n_q, s->n_k, s->H_I, s->d_I, s->topk, s->qk_dtype, &a);
    if (st != IC_OK) return st;
    st = ic_sparse_attn_workspace_size(s->batch, s->n_q, s->H, s->d_v, s->topk, &b);
    if (st != IC_OK) return st;
    *bytes_out = std::max(a, b);
    return IC_OK;
}

ic_status ic_layer_stack(const ic_layer_io* layers, int n_layers, int index_topk_freq,
                         const char* index_topk_pattern, const ic_stack_shape* s, int32_t* idx_buffer,
                         void* workspace, size_t workspace_bytes, void* stream) {
    if (!layers || !s || !idx_buffer) return IC_ERR_INVALID_ARG;
    std::vector<uint8_t> is_full(static_cast<size_t>(std::max(n_layers, 1)));
    std::vector<int32_t> src(static_cast<size_t>(std::max(n_layers, 1)));
    ic_status st = ic_resolve_pattern(n_layers, index_topk_freq, index_topk_pattern, is_full.data(), src.data());
    if (st != IC_OK) return st;
    // validate every layer before enqueueing anything
    for (int l = 0; l < n_layers; ++l) {
        const ic_layer_io& L = layers[l];
        if (is_full[l]) {
            st = validate_indexer(L.q_I, L.q_scale, L.w, s->w_dtype, L.k_I, L.k_scale, s->qk_dtype, s->batch, s->n_q,
                                  s->n_k, s->q_pos0, s->H_I, s->d_I, s->topk, idx_buffer);
            if (st != IC_OK) return st;
        }
        if (s->batch > 0 && s->n_q > 0 && (!L.q || !L.out || (s->n_k > 0 && !L.kv))) return IC_ERR_INVALID_ARG;
    }
    const cudaStream_t cs = static_cast<cudaStream_t>(stream);
    // every launch after the call's first follows one of this library's
    // kernels: it may start while that one finishes (programmatic dependency)
    bool pdl = false;
    for (int l = 0; l < n_layers; ++l) {
        const ic_layer_io& L = layers[l];
        if (is_full[l]) {  // the single conditional branch: Full layers refresh the cached indices
            st = launch_indexer(L.q_I, L.q_scale, L.w, s->w_dtype, L.k_I, L.k_scale, s->qk_dtype, s->batch, s->n_q,
                                s->n_k, s->q_pos0, s->H_I, s->d_I, s->topk, idx_buffer, workspace, workspace_bytes,
                                cs, true, pdl);
            if (st != IC_OK) return st;
            pdl = true;
        }
        st = launch_attn(L.q, L.kv, idx_buffer, s->batch, s->n_q, s->n_k, s->H, s->d_qk, s->d_v, s->topk, s->sm_scale,
                         L.out, workspace, workspace_bytes, cs, pdl);
        if (st != IC_OK) return st;
        pdl = true;
    }
    return IC_OK;
}

// ---------------------------------------------------------------------------
// Layer loop over host-resident tensors: two device slots, copies on two
// internal streams overlapping the kernels on the caller's stream.
// ---------------------------------------------------------------------------
namespace {

// Fields of ic_layer_io in declaration order; the last one is the output.
enum HostField { HF_QI, HF_QSCALE, HF_W, HF_KI, HF_KSCALE, HF_Q, HF_KV, HF_OUT, HF_COUNT };

const void* field_ptr(const ic_layer_io& L, int f) {
    switch (f) {
        case HF_QI: return L.q_I;
        case HF_QSCALE: return L.q_scale;
        case HF_W: return L.w;
        case HF_KI: return L.k_I;
        case HF_KSCALE: return L.k_scale;
        case HF_Q: return L.q;
        case HF_KV: return L.kv;
        default: return L.out;
    }
}

// Bytes of each field for one layer of the shape.
void field_bytes(const ic_stack_shape& s, size_t out[HF_COUNT]) {
    const size_t B = static_cast<size_t>(s.batch), nq = static_cast<size_t>(s.n_q), nk = static_cast<size_t>(s.n_k);
    const size_t qk = s.qk_dtype == IC_FP8_E4M3 ? 1 : 2, wsz = s.w_dtype == IC_F32 ? 4 : 2;
    out[HF_QI] = B * nq * s.H_I * s.d_I * qk;
    out[HF_QSCALE] = B * nq * 4;
    out[HF_W] = B * nq * s.H_I * wsz;
    out[HF_KI] = B * nk * s.d_I * qk;
    out[HF_KSCALE] = B * nk * 4;
    out[HF_Q] = B * nq * s.H * s.d_qk * 2;
    out[HF_KV] = B * nk * s.d_qk * 2;
    out[HF_OUT] = B * nq * s.H * s.d_v * 2;
}

// True when p is host memory (page-locked or pageable); device and managed
// memory are used in place. A pointer CUDA does not know is host memory.
bool is_host_memory(const void* p) {
    if (p == nullptr) return false;
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        (void)cudaGetLastError();
        return true;
    }
    return a.type == cudaMemoryTypeHost || a.type == cudaMemoryTypeUnregistered;
}

// Which fields any layer passes in host memory, and the staging layout:
// slot 0 and slot 1 (one offset per staged field), the index buffer, the
// workspace.
struct HostPlan {
    bool staged[HF_COUNT] = {};
    size_t field[HF_COUNT] = {};
    size_t off[HF_COUNT] = {};
    size_t slot_bytes = 0, off_idx = 0, off_ws = 0, ws_bytes = 0, total = 0;
};

ic_status host_plan(const ic_layer_io* layers, int n_layers, const ic_stack_shape& s, HostPlan* hp) {
    field_bytes(s, hp->field);
    for (int l = 0; l < n_layers; ++l)
        for (int f = 0; f < HF_COUNT; ++f)
            if (is_host_memory(field_ptr(layers[l], f))) hp->staged[f] = true;
    size_t o = 0;
    for (int f = 0; f < HF_COUNT; ++f) {
        hp->off[f] = o;
        if (hp->staged[f]) o += round_up(hp->field[f], 256);
    }
    hp->slot_bytes = o;
    hp->off_idx = 2 * o;
    const size_t idx_bytes = static_cast<size_t>(s.batch) * s.n_q * s.topk * 4;
    hp->off_ws = hp->off_idx + round_up(idx_bytes, 256);
    ic_status st = ic_layer_stack_workspace_size(&s, &hp->ws_bytes);
    if (st != IC_OK) return st;
    hp->total = hp->off_ws + round_up(hp->ws_bytes, 256);
    return IC_OK;
}

struct CopyStreams {
    cudaStream_t h2d = nullptr, d2h = nullptr;
};

// The two copy streams of a device, created on first use and kept.
ic_status copy_streams(int dev, CopyStreams* out) {
    static std::mutex mu;
    static std::vector<CopyStreams> per_dev;
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 0) return IC_ERR_INVALID_ARG;
    if (per_dev.size() <= static_cast<size_t>(dev)) per_dev.resize(static_cast<size_t>(dev) + 1);
    CopyStreams& c = per_dev[static_cast<size_t>(dev)];
    if (c.h2d == nullptr) {
        cudaError_t e = cudaStreamCreateWithFlags(&c.h2d, cudaStreamNonBlocking);
        if (e != cudaSuccess) return cuda_fail("copy stream", e);
        e = cudaStreamCreateWithFlags(&c.d2h, cudaStreamNonBlocking);
        if (e != cudaSuccess) return cuda_fail("copy stream", e);
    }
    *out = c;
    return IC_OK;
}

// Events of one call, destroyed when the call returns (CUDA releases each
// one once its recorded work has completed).
struct CallEvents {
    static constexpr int N = 9;  // start, in[2], done[2], out[2], h2d end, d2h end
    cudaEvent_t e[N] = {};
    ~CallEvents() {
        for (cudaEvent_t x : e)
            if (x) cudaEventDestroy(x);
    }
    ic_status create() {
        for (cudaEvent_t& x : e) {
            const cudaError_t r = cudaEventCreateWithFlags(&x, cudaEventDisableTiming);
            if (r != cudaSuccess) return cuda_fail("event", r);
        }
        return IC_OK;
    }
};

}  // namespace

ic_status ic_layer_stack_host_staging_size(const ic_layer_io* layers, int n_layers, const ic_stack_shape* s,
                                           size_t* bytes_out) {
    if (!layers || !s || !bytes_out || n_layers < 1) return IC_ERR_INVALID_ARG;
    HostPlan hp;
    const ic_status st = host_plan(layers, n_layers, *s, &hp);
    if (st != IC_OK) return st;
    *bytes_out = hp.total;
    return IC_OK;
}

ic_status ic_layer_stack_host(const ic_layer_io* layers, int n_layers, int index_topk_freq,
                              const char* index_topk_pattern, const ic_stack_shape* s, int32_t* idx_host_out,
                              void* staging, size_t staging_bytes, void* stream, size_t* h2d_bytes_out,
                              size_t* d2h_bytes_out) {
    if (!layers || !s) return IC_ERR_INVALID_ARG;
    std::vector<uint8_t> is_full(static_cast<size_t>(std::max(n_layers, 1)));
    std::vector<int32_t> src(static_cast<size_t>(std::max(n_layers, 1)));
    ic_status st = ic_resolve_pattern(n_layers, index_topk_freq, index_topk_pattern, is_full.data(), src.data());
    if (st != IC_OK) return st;
    // A host output that overlaps a host input could be copied out after a
    // later layer's copy of that input has already been taken: refused.
    {
        size_t fb[HF_COUNT];
        field_bytes(*s, fb);
        struct Range { uintptr_t lo, hi; };
        std::vector<Range> ins, outs;
        for (int l = 0; l < n_layers; ++l) {
            for (int f = 0; f < HF_COUNT; ++f) {
                const void* h = field_ptr(layers[l], f);
                if (h == nullptr || fb[f] == 0 || !(f >= HF_Q || is_full[l]) || !is_host_memory(h)) continue;
                const Range r{reinterpret_cast<uintptr_t>(h), reinterpret_cast<uintptr_t>(h) + fb[f]};
                (f == HF_OUT ? outs : ins).push_back(r);
            }
        }
        for (const Range& o : outs)
            for (const Range& i : ins)
                if (o.lo < i.hi && i.lo < o.hi) return IC_ERR_INVALID_ARG;
    }
    HostPlan hp;
    st = host_plan(layers, n_layers, *s, &hp);
    if (st != IC_OK) return st;
    if (!staging || !aligned256(staging) || staging_bytes < hp.total) return IC_ERR_WORKSPACE;
    uint8_t* base = static_cast<uint8_t*>(staging);
    int32_t* idx_dev = reinterpret_cast<int32_t*>(base + hp.off_idx);
    void* ws = hp.ws_bytes ? base + hp.off_ws : nullptr;

    // the device view of every layer (staged fields point into the layer's
    // slot) and which of its fields are copied; validated before any enqueue.
    // A host input that the slot already holds (the same buffer staged there
    // by layer l-2 or earlier, and not overwritten since) is not copied again.
    std::vector<ic_layer_io> dv(static_cast<size_t>(n_layers));
    std::vector<uint16_t> copy_mask(static_cast<size_t>(n_layers), 0);
    const void* held[2][HF_COUNT] = {};
    size_t h2d = 0, d2h = 0;
    for (int l = 0; l < n_layers; ++l) {
        const ic_layer_io& H = layers[l];
        uint8_t* slot = base + static_cast<size_t>(l & 1) * hp.slot_bytes;
        const void* p[HF_COUNT];
        for (int f = 0; f < HF_COUNT; ++f) {
            const void* h = field_ptr(H, f);
            const bool used = f >= HF_Q || is_full[l];
            p[f] = h;
            if (used && h != nullptr && hp.staged[f] && is_host_memory(h)) {
                p[f] = slot + hp.off[f];
                if (f == HF_OUT) {
                    copy_mask[l] |= static_cast<uint16_t>(1u << f);
                    d2h += hp.field[f];
                } else if (held[l & 1][f] != h) {
                    copy_mask[l] |= static_cast<uint16_t>(1u << f);
                    held[l & 1][f] = h;
                    h2d += hp.field[f];
                }
            }
        }
        ic_layer_io& D = dv[l];
        D.q_I = p[HF_QI];
        D.q_scale = static_cast<const float*>(p[HF_QSCALE]);
        D.w = p[HF_W];
        D.k_I = p[HF_KI];
        D.k_scale = static_cast<const float*>(p[HF_KSCALE]);
        D.q = p[HF_Q];
        D.kv = p[HF_KV];
        D.out = const_cast<void*>(p[HF_OUT]);
        if (is_full[l]) {
            st = validate_indexer(D.q_I, D.q_scale, D.w, s->w_dtype, D.k_I, D.k_scale, s->qk_dtype, s->batch, s->n_q,
                                  s->n_k, s->q_pos0, s->H_I, s->d_I, s->topk, idx_dev);
            if (st != IC_OK) return st;
        }
        if (s->batch > 0 && s->n_q > 0 && (!D.q || !D.out || (s->n_k > 0 && !D.kv))) return IC_ERR_INVALID_ARG;
    }

    if (idx_host_out != nullptr) d2h += static_cast<size_t>(s->batch) * s->n_q * s->topk * 4;
    if (h2d_bytes_out) *h2d_bytes_out = h2d;
    if (d2h_bytes_out) *d2h_bytes_out = d2h;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail("device", e);
    CopyStreams cp;
    st = copy_streams(dev, &cp);
    if (st != IC_OK) return st;
    CallEvents ev;
    st = ev.create();
    if (st != IC_OK) return st;
    cudaEvent_t& ev_start = ev.e[0];
    cudaEvent_t* ev_in = ev.e + 1;
    cudaEvent_t* ev_done = ev.e + 3;
    cudaEvent_t* ev_out = ev.e + 5;
    cudaEvent_t& ev_h2d_end = ev.e[7];
    cudaEvent_t& ev_d2h_end = ev.e[8];
    const cudaStream_t cs = static_cast<cudaStream_t>(stream);
    auto ok = [](cudaError_t r, const char* what) { return r == cudaSuccess ? IC_OK : cuda_fail(what, r); };

    // fork the copy streams from the caller's stream
    if ((st = ok(cudaEventRecord(ev_start, cs), "event record")) != IC_OK) return st;
    if ((st = ok(cudaStreamWaitEvent(cp.h2d, ev_start, 0), "stream wait")) != IC_OK) return st;
    if ((st = ok(cudaStreamWaitEvent(cp.d2h, ev_start, 0), "stream wait")) != IC_OK) return st;
    for (int l = 0; l < n_layers; ++l) {
        const int sl = l & 1;
        const ic_layer_io& H = layers[l];
        const ic_layer_io& D = dv[l];
        const bool out_staged = (copy_mask[l] >> HF_OUT) & 1u;
        // inputs of layer l into its slot, once layer l-2 no longer reads it
        if (l >= 2 && (st = ok(cudaStreamWaitEvent(cp.h2d, ev_done[sl], 0), "stream wait")) != IC_OK) return st;
        for (int f = 0; f < HF_OUT; ++f) {
            if (!((copy_mask[l] >> f) & 1u)) continue;
            const void* dst = field_ptr(D, f);
            e = cudaMemcpyAsync(const_cast<void*>(dst), field_ptr(H, f), hp.field[f], cudaMemcpyHostToDevice, cp.h2d);
            if (e != cudaSuccess) return cuda_fail("input copy", e);
        }
        if ((st = ok(cudaEventRecord(ev_in[sl], cp.h2d), "event record")) != IC_OK) return st;
        // the layer's kernels, once its inputs are in and the slot's previous
        // output has been copied out
        if ((st = ok(cudaStreamWaitEvent(cs, ev_in[sl], 0), "stream wait")) != IC_OK) return st;
        if (l >= 2 && (st = ok(cudaStreamWaitEvent(cs, ev_out[sl], 0), "stream wait")) != IC_OK) return st;
        if (is_full[l]) {
            st = launch_indexer(D.q_I, D.q_scale, D.w, s->w_dtype, D.k_I, D.k_scale, s->qk_dtype, s->batch, s->n_q,
                                s->n_k, s->q_pos0, s->H_I, s->d_I, s->topk, idx_dev, ws, hp.ws_bytes, cs);
            if (st != IC_OK) return st;
        }
        st = launch_attn(D.q, D.kv, idx_dev, s->batch, s->n_q, s->n_k, s->H, s->d_qk, s->d_v, s->topk, s->sm_scale,
                         D.out, ws, hp.ws_bytes, cs);
        if (st != IC_OK) return st;
        if ((st = ok(cudaEventRecord(ev_done[sl], cs), "event record")) != IC_OK) return st;
        // the output back to the host
        if ((st = ok(cudaStreamWaitEvent(cp.d2h, ev_done[sl], 0), "stream wait")) != IC_OK) return st;
        if (out_staged) {
            e = cudaMemcpyAsync(H.out, D.out, hp.field[HF_OUT], cudaMemcpyDeviceToHost, cp.d2h);
            if (e != cudaSuccess) return cuda_fail("output copy", e);
        }
        if ((st = ok(cudaEventRecord(ev_out[sl], cp.d2h), "event record")) != IC_OK) return st;
    }
    if (idx_host_out != nullptr && s->batch > 0 && s->n_q > 0) {
        e = cudaMemcpyAsync(idx_host_out, idx_dev, static_cast<size_t>(s->batch) * s->n_q * s->topk * 4,
                            cudaMemcpyDefault, cp.d2h);
        if (e != cudaSuccess) return cuda_fail("index copy", e);
    }
    // join the copy streams back into the caller's stream
    if ((st = ok(cudaEventRecord(ev_h2d_end, cp.h2d), "event record")) != IC_OK) return st;
    if ((st = ok(cudaEventRecord(ev_d2h_end, cp.d2h), "event record")) != IC_OK) return st;
    if ((st = ok(cudaStreamWaitEvent(cs, ev_h2d_end, 0), "stream wait")) != IC_OK) return st;
    if ((st = ok(cudaStreamWaitEvent(cs, ev_d2h_end, 0), "stream wait")) != IC_OK) return st;
    return IC_OK;
}


ic_status ic_distill_target_workspace_size(int batch, int n_q, int topk, int H, int d_qk, int H_I, int d_I,
                                           size_t* bytes_out) {
    if (!bytes_out || batch < 0 || n_q < 0 || topk <= 0 || H <= 0 || d_qk <= 0 || H_I <= 0 || d_I <= 0)
        return IC_ERR_INVALID_ARG;
    if (static_cast<int64_t>(batch) * n_q > std::numeric_limits<int>::max()) return IC_ERR_UNSUPPORTED;
    *bytes_out = 0;
    if (!distill_on_tensor_cores(H, d_qk, H_I, d_I) || topk > 2048) return IC_OK;
    const DeviceInfo dev = device_info();
    if (dev.sms <= 0) return cuda_fail("device query", cudaErrorNoDevice);
    *bytes_out = distill_tc_ws_bytes(batch * n_q, topk, dev.sms);
    return IC_OK;
}

ic_status ic_distill_target(const void* const* q_layers, const void* const* kv_layers, int n_served,
                            const void* q_I, const float* q_scale, const void* w, ic_dtype w_dtype,
                            const void* k_I, const float* k_scale, ic_dtype qk_dtype, const int32_t* idx,
                            int batch, int n_q, int n_k, int H_I, int d_I, int topk, int H, int d_qk,
                            float sm_scale, float* target_out, float* kl_out, void* workspace,
                            size_t workspace_bytes, void* stream) {
    if (batch < 0 || n_q < 0 || n_k < 0 || topk <= 0 || H <= 0 || d_qk <= 0 || H_I <= 0 || d_I <= 0)
        return IC_ERR_INVALID_ARG;
    if (n_served < 1 || !q_layers || !kv_layers) return IC_ERR_INVALID_ARG;
    if (qk_dtype != IC_BF16 && qk_dtype != IC_FP8_E4M3) return IC_ERR_INVALID_ARG;
    if (w_dtype != IC_BF16 && w_dtype != IC_F32) return IC_ERR_INVALID_ARG;
    if (n_served > ic::DISTILL_MAX_SERVED || (d_qk != 64 && d_qk != 576) || H > 64 || (H_I != 4 && H_I != 64) ||
        d_I % 8 != 0 || d_I > 128 || topk > 2048)
        return IC_ERR_UNSUPPORTED;
    if (static_cast<int64_t>(batch) * n_q > std::numeric_limits<int>::max()) return IC_ERR_UNSUPPORTED;
    if (batch == 0 || n_q == 0) return IC_OK;
    if (!q_I || !w || !idx || !kl_out || (n_k > 0 && !k_I)) return IC_ERR_INVALID_ARG;
    if (qk_dtype == IC_FP8_E4M3 && (!q_scale || (n_k > 0 && !k_scale))) return IC_ERR_INVALID_ARG;
    if (!aligned16(k_I) || !aligned16(q_I)) return IC_ERR_INVALID_ARG;
    ic::DistillParams p{};
    for (int l = 0; l < n_served; ++l) {
        if (!q_layers[l] || (n_k > 0 && !kv_layers[l])) return IC_ERR_INVALID_ARG;
        if (!aligned16(q_layers[l]) || !aligned16(kv_layers[l])) return IC_ERR_INVALID_ARG;
        p.q[l] = static_cast<const __nv_bfloat16*>(q_layers[l]);
        p.kv[l] = static_cast<const __nv_bfloat16*>(kv_layers[l]);
    }
    p.n_served = n_served;
    p.q_I = q_I;
    p.q_scale = q_scale;
    p.w = w;
    p.w_is_f32 = w_dtype == IC_F32 ? 1 : 0;
    p.k_I = k_I;
    p.k_scale = k_scale;
    p.fp8 = qk_dtype == IC_FP8_E4M3 ? 1 : 0;
    p.idx = idx;
    p.n_q = n_q;
    p.n_k = n_k;
    p.topk = topk;
    p.H = H;
    p.d_I = d_I;
    p.sm_scale = sm_scale;
    p.target = target_out;
    p.kl = kl_out;
    const int rows = batch * n_q;
    p.rows = rows;
    const cudaStream_t cs = static_cast<cudaStream_t>(stream);
    // the model's shapes (64 heads over 576-wide latent rows, a 64-head
    // 128-wide indexer) run on the tensor cores; other shapes on the CUDA cores
    if (distill_on_tensor_cores(H, d_qk, H_I, d_I)) {
        const DeviceInfo dev = device_info();
        if (dev.sms <= 0) return cuda_fail("device query", cudaErrorNoDevice);
        const size_t need = distill_tc_ws_bytes(rows, topk, dev.sms);
        if (need > 0 && (!workspace || workspace_bytes < need || !aligned256(workspace))) return IC_ERR_WORKSPACE;
        p.spill = workspace;
        return p.fp8 ? launch_distill_tc<ic::DistTcCfg<576, true>>(p, dev.sms, cs)
                     : launch_distill_tc<ic::DistTcCfg<576, false>>(p, dev.sms, cs);
    }
    if (d_qk == 576) return H_I == 64 ? launch_distill<576, 64>(p, rows, cs) : launch_distill<576, 4>(p, rows, cs);
    return H_I == 64 ? launch_distill<64, 64>(p, rows, cs) : launch_distill<64, 4>(p, rows, cs);
}

ic_status ic_get_device_status(int reset) {
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail("synchronize", e);
    int v = 0;
    e = cudaMemcpyFromSymbol(&v, ic::g_device_status, sizeof(int));
    if (e != cudaSuccess) return cuda_fail("read device status", e);
    if (reset) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(ic::g_device_status, &zero, sizeof(int));
        if (e != cudaSuccess) return cuda_fail("reset device status", e);
    }
    return static_cast<ic_status>(v);
}

ic_status ic_debug_expire_wait(long long timeout_ns, void* stream) {
    if (timeout_ns <= 0 || timeout_ns > 10000000000LL) return IC_ERR_INVALID_ARG;
    expire_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(timeout_ns);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? IC_OK : cuda_fail("expire-wait launch", e);
}

const char* ic_last_error_string(void) { return g_last_error; }

ic_status ic_indexer_topk_noalloc(const void* q_I, const float* q_scale, const void* w, ic_dtype w_dtype,
                                  const void* k_I, const float* k_scale, ic_dtype qk_dtype, int batch, int n_q,
                                  int n_k, int q_pos0, int H_I, int d_I, int topk, int32_t* idx_out,
                                  void* stream) {
    ic_status st = validate_indexer(q_I, q_scale, w, w_dtype, k_I, k_scale, qk_dtype, batch, n_q, n_k, q_pos0, H_I,
                                    d_I, topk, idx_out);
    if (st != IC_OK) return st;
    if (batch == 0 || n_q == 0) return IC_OK;
    IdxPlan pl;
    if (!choose_idx_plan(H_I, d_I, qk_dtype, n_q, &pl) || !plan_supports_topk(pl, topk)) return IC_ERR_UNSUPPORTED;
    const DeviceInfo dev = device_info();
    if (dev.sms <= 0) return cuda_fail("device query", cudaErrorNoDevice);
    // the split candidate lists, not the decode score rows: their size does
    // not grow with the number of visible keys
    const size_t need = idx_layout(pl, batch, n_q, n_k, topk, dev.sms, false).bytes;
    if (need > IC_NOALLOC_SCRATCH_BYTES) {
        std::snprintf(g_last_error, sizeof g_last_error,
                      "ic_indexer_topk_noalloc: needs %zu bytes of scratch, the fixed array holds %u",
                      need, IC_NOALLOC_SCRATCH_BYTES);
        return IC_ERR_WORKSPACE;
    }
    void* scratch = nullptr;
    if (need > 0) {
        st = noalloc_scratch(&scratch);
        if (st != IC_OK) return st;
    }
    // The split path writes every candidate count before the merge reads it,
    // so nothing in the scratch has to start at zero.
    return launch_indexer(q_I, q_scale, w, w_dtype, k_I, k_scale, qk_dtype, batch, n_q, n_k, q_pos0, H_I, d_I, topk,
                          idx_out, scratch, need > 0 ? IC_NOALLOC_SCRATCH_BYTES : 0,
                          static_cast<cudaStream_t>(stream), false);
}

ic_status ic_indexer_noalloc_scratch_size(int batch, int n_q, int n_k, int H_I, int d_I, int topk, ic_dtype qk_dtype,
                                          size_t* bytes_out) {
    if (!bytes_out || batch < 0 || n_q < 0 || n_k < 0 || topk <= 0) return IC_ERR_INVALID_ARG;
    *bytes_out = 0;
    if (batch == 0 || n_q == 0) return IC_OK;
    IdxPlan pl;
    if (!choose_idx_plan(H_I, d_I, qk_dtype, n_q, &pl) || !plan_supports_topk(pl, topk)) return IC_ERR_UNSUPPORTED;
    const DeviceInfo dev = device_info();
    if (dev.sms <= 0) return cuda_fail("device query", cudaErrorNoDevice);
    *bytes_out = idx_layout(pl, batch, n_q, n_k, topk, dev.sms, false).bytes;
    return IC_OK;
}

size_t ic_indexer_noalloc_max_scratch(void) { return IC_NOALLOC_SCRATCH_BYTES; }

}  // extern "C"
