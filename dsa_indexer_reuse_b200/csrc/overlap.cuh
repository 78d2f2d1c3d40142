// Pairwise top-k overlap of two index buffers (IndexCache paper, Appendix
// Figure 4: the pairwise top-k index overlap ratio between layer pairs, which
// motivates sharing one layer's indices with its neighbours).
//
//     counts[r] = | {valid entries of a[r]} intersect {valid entries of b[r]} |
//
// for index rows as ic_indexer_topk writes them (entries in [0, n_k) are
// valid, anything else is padding; no index repeats within a row). The result
// does not depend on the order of a row's entries.
//
// One persistent CTA per SM walks rows; each keeps an n_k-bit set in shared
// memory: it marks row a's entries, tests row b's, reduces the hit count, and
// clears exactly the words it marked before the next row.
#pragma once

#include "common.cuh"

namespace ic {

constexpr int OVERLAP_THREADS = 256;

__global__ void __launch_bounds__(OVERLAP_THREADS)
    topk_overlap_kernel(const int32_t* __restrict__ a, const int32_t* __restrict__ b, int rows, int topk, int n_k,
                        int32_t* __restrict__ counts) {
    extern __shared__ uint32_t bits[];
    __shared__ int warp_sum[OVERLAP_THREADS / 32];
    const int tid = threadIdx.x;
    const int nwords = (n_k + 31) / 32;
    for (int i = tid; i < nwords; i += OVERLAP_THREADS) bits[i] = 0u;
    __syncthreads();
    for (int row = blockIdx.x; row < rows; row += gridDim.x) {
        const int32_t* ra = a + static_cast<int64_t>(row) * topk;
        const int32_t* rb = b + static_cast<int64_t>(row) * topk;
        for (int i = tid; i < topk; i += OVERLAP_THREADS) {
            const int v = ra[i];
            if (v >= 0 && v < n_k) atomicOr(&bits[v >> 5], 1u << (v & 31));
        }
        __syncthreads();
        int c = 0;
        for (int i = tid; i < topk; i += OVERLAP_THREADS) {
            const int v = rb[i];
            if (v >= 0 && v < n_k) c += (bits[v >> 5] >> (v & 31)) & 1u;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
        if ((tid & 31) == 0) warp_sum[tid >> 5] = c;
        __syncthreads();
        if (tid == 0) {
            int s = 0;
#pragma unroll
            for (int w = 0; w < OVERLAP_THREADS / 32; ++w) s += warp_sum[w];
            counts[row] = s;
        }
        // clear the words this row marked (every writer stores 0)
        for (int i = tid; i < topk; i += OVERLAP_THREADS) {
            const int v = ra[i];
            if (v >= 0 && v < n_k) bits[v >> 5] = 0u;
        }
        __syncthreads();
    }
}

// All pairwise overlap counts of one layer's index buffer against every
// layer's (the rows of the overlap matrix for layer a):
//     counts[a * n_layers + b] += sum over rows of |valid(T_a[r]) & valid(T_b[r])|
// (the diagonal is layer a's valid-entry count). Same per-row key set as
// topk_overlap_kernel: row a's entries are marked once and every layer's row
// is tested against them. Each CTA sums its rows per layer in shared memory
// and adds the sums to `counts` once at the end.
constexpr int OVERLAP_MAX_LAYERS = 128;

struct OverlapLayers {
    const int32_t* p[OVERLAP_MAX_LAYERS];
};

__global__ void __launch_bounds__(OVERLAP_THREADS)
    overlap_counts_kernel(const OverlapLayers L, int a, int n_layers, int rows, int topk, int n_k,
                          unsigned long long* __restrict__ counts) {
    extern __shared__ uint32_t bits[];
    __shared__ unsigned long long sums[OVERLAP_MAX_LAYERS];
    __shared__ int warp_sum[OVERLAP_THREADS / 32];
    const int tid = threadIdx.x;
    const int nwords = (n_k + 31) / 32;
    for (int i = tid; i < nwords; i += OVERLAP_THREADS) bits[i] = 0u;
    for (int i = tid; i < n_layers; i += OVERLAP_THREADS) sums[i] = 0ull;
    __syncthreads();
    const int32_t* A = L.p[a];
    for (int row = blockIdx.x; row < rows; row += gridDim.x) {
        const int32_t* ra = A + static_cast<int64_t>(row) * topk;
        for (int i = tid; i < topk; i += OVERLAP_THREADS) {
            const int v = ra[i];
            if (v >= 0 && v < n_k) atomicOr(&bits[v >> 5], 1u << (v & 31));
        }
        __syncthreads();
        for (int b = 0; b < n_layers; ++b) {
            const int32_t* rb = L.p[b] + static_cast<int64_t>(row) * topk;
            int c = 0;
            for (int i = tid; i < topk; i += OVERLAP_THREADS) {
                const int v = rb[i];
                if (v >= 0 && v < n_k) c += (bits[v >> 5] >> (v & 31)) & 1u;
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
            if ((tid & 31) == 0) warp_sum[tid >> 5] = c;
            __syncthreads();
            if (tid == 0) {
                int s = 0;
#pragma unroll
                for (int w = 0; w < OVERLAP_THREADS / 32; ++w) s += warp_sum[w];
                sums[b] += static_cast<unsigned long long>(s);
            }
            __syncthreads();
        }
        // clear the words this row marked (every writer stores 0)
        for (int i = tid; i < topk; i += OVERLAP_THREADS) {
            const int v = ra[i];
            if (v >= 0 && v < n_k) bits[v >> 5] = 0u;
        }
        __syncthreads();
    }
    for (int b = tid; b < n_layers; b += OVERLAP_THREADS)
        if (sums[b] != 0ull) atomicAdd(&counts[static_cast<int64_t>(a) * n_layers + b], sums[b]);
}

}  // namespace ic
