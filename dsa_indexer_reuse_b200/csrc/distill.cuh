// Multi-layer distillation target (IndexCache paper, Abstract: each retained
// indexer is trained against the averaged attention distributions of all the
// layers it serves; Table 3, "w/o cross-layer loss": each indexer against its
// own layer only). Forward quantities only; training is not part of this
// library. For query row r and the positions j of the Full layer's index row
// whose key s_j lies in [0, n_k):
//   P[j]  = (1 / (n_served * H)) sum_l sum_h softmax_j(sm_scale * q_l[r,h,:] . kv_l[s_j,:])
//   Q[j]  = softmax_j(I[r, s_j])   (the Full layer's indexer score at those keys)
//   kl[r] = sum_j P[j] * (log P[j] - log Q[j])
// target[r][j] = P[j] (0 at invalid positions); a row with no valid position
// has an all-zero target and kl 0.
//
// One 256-thread CTA per query row. For each served layer, heads are taken 16
// at a time: every thread computes the 16 logits of its keys (fp32 packed
// FMAs against the group's q rows, held as fp32 in shared memory) and keeps
// them in shared memory, with a running (max, sum of exp) per head; a block
// reduction of those pairs gives each head's softmax normaliser, and one pass
// over the stored logits adds the group's probabilities into P. The indexer
// scores of the same keys follow, then the softmax and the KL, each as a
// block reduction. The work is CUDA-core arithmetic: per row and served layer
// it is topk * H * d_qk multiply-adds, with the key rows read from L2.
#pragma once

#include <cuda_fp8.h>

#include "common.cuh"

namespace ic {

constexpr int DISTILL_MAX_SERVED = 64;
constexpr int DISTILL_THREADS = 256;
constexpr int DISTILL_HG = 16;  // heads per group

struct DistillParams {
    const __nv_bfloat16* q[DISTILL_MAX_SERVED];   // served layers' q  [batch, n_q, H, d_qk]
    const __nv_bfloat16* kv[DISTILL_MAX_SERVED];  // served layers' kv [batch, n_k, d_qk]
    int n_served;
    const void* q_I;        // Full layer's indexer tensors, as in IdxParams
    const float* q_scale;
    const void* w;
    int w_is_f32;
    const void* k_I;
    const float* k_scale;
    int fp8;
    const int32_t* idx;     // [batch * n_q, topk]
    int n_q, n_k, topk, H, d_I;
    int rows;               // batch * n_q
    void* spill;            // tensor-core kernel: per-CTA logit workspace
    float sm_scale;
    float* target;          // [batch * n_q, topk] or null
    float* kl;              // [batch * n_q]
};

// Shared-memory floats of one CTA (the logits of a head group, the q rows of
// the group or the indexer query, P, the key list, per-head weights and the
// reduction scratch).
__host__ __device__ constexpr int distill_qf_floats(int dqk, int hi, int d_i) {
    return DISTILL_HG * dqk > hi * d_i ? DISTILL_HG * dqk : hi * d_i;
}
__host__ __device__ constexpr size_t distill_smem_bytes(int dqk, int hi, int d_i, int topk) {
    return 4ull * (static_cast<size_t>(DISTILL_HG) * topk + distill_qf_floats(dqk, hi, d_i) + 2ull * topk + 64 +
                   2 * (DISTILL_THREADS / 32) * DISTILL_HG + 2 * DISTILL_HG + 8);
}

__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t v) {
    return make_float2(__uint_as_float(v << 16), __uint_as_float(v & 0xFFFF0000u));
}

// Merge two (max, sum of exp relative to max) pairs.
__device__ __forceinline__ void ml_merge(float& m, float& l, float m2, float l2) {
    const float mm = fmaxf(m, m2);
    if (mm == -INFINITY) return;  // both empty
    l = l * expf(m - mm) + l2 * expf(m2 - mm);
    m = mm;
}

__device__ __forceinline__ float block_sum(float v, float* scratch) {
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0) scratch[warp] = v;
    __syncthreads();
    float t = 0.f;
    for (int w = 0; w < DISTILL_THREADS / 32; ++w) t += scratch[w];
    return t;
}

__device__ __forceinline__ float block_max(float v, float* scratch) {
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0) scratch[warp] = v;
    __syncthreads();
    float t = -INFINITY;
    for (int w = 0; w < DISTILL_THREADS / 32; ++w) t = fmaxf(t, scratch[w]);
    return t;
}

template <int DQK, int HI>
__global__ void __launch_bounds__(DISTILL_THREADS, 1) distill_target_kernel(const __grid_constant__ DistillParams p) {
    static_assert(DQK % 8 == 0, "d_qk");
    constexpr int NW = DISTILL_THREADS / 32;
    extern __shared__ float dsm[];
    const int topk = p.topk;
    float* zs = dsm;                                            // [HG][topk] logits
    float* qf = zs + DISTILL_HG * topk;                         // q rows of a group / indexer query
    float* P = qf + distill_qf_floats(DQK, HI, p.d_I);          // [topk] target
    int* keys = reinterpret_cast<int*>(P + topk);               // [topk] key or -1
    float* wq = reinterpret_cast<float*>(keys + topk);          // [64] w * q_scale
    float* red_m = wq + 64;                                     // [NW][HG]
    float* red_l = red_m + NW * DISTILL_HG;                     // [NW][HG]
    float* head_m = red_l + NW * DISTILL_HG;                    // [HG]
    float* head_l = head_m + DISTILL_HG;                        // [HG]
    float* scratch = head_l + DISTILL_HG;                       // [8]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t row = blockIdx.x;
    const int b = static_cast<int>(row / p.n_q);
    int n_valid = 0;
    for (int j = tid; j < topk; j += DISTILL_THREADS) {
        const int s = p.idx[row * topk + j];
        const bool ok = s >= 0 && s < p.n_k;
        keys[j] = ok ? s : -1;
        P[j] = 0.f;
        n_valid += ok ? 1 : 0;
    }
    n_valid = static_cast<int>(block_sum(static_cast<float>(n_valid), scratch));
    if (n_valid == 0) {
        for (int j = tid; j < topk; j += DISTILL_THREADS)
            if (p.target) p.target[row * topk + j] = 0.f;
        if (tid == 0) p.kl[row] = 0.f;
        return;
    }
    const float inv_norm = 1.f / (static_cast<float>(p.H) * static_cast<float>(p.n_served));

    // ---- the target: head- and layer-averaged attention probabilities
    for (int l = 0; l < p.n_served; ++l) {
        const __nv_bfloat16* qrow = p.q[l] + row * p.H * DQK;
        const __nv_bfloat16* kvb = p.kv[l] + static_cast<int64_t>(b) * p.n_k * DQK;
        for (int h0 = 0; h0 < p.H; h0 += DISTILL_HG) {
            const int hgn = min(DISTILL_HG, p.H - h0);
            __syncthreads();  // qf, zs and the head stats are reused
            for (int i = tid; i < hgn * DQK; i += DISTILL_THREADS)
                qf[i] = __bfloat162float(qrow[h0 * DQK + i]);
            __syncthreads();
            float m[DISTILL_HG], lsum[DISTILL_HG];
#pragma unroll
            for (int h = 0; h < DISTILL_HG; ++h) {
                m[h] = -INFINITY;
                lsum[h] = 0.f;
            }
            for (int j = tid; j < topk; j += DISTILL_THREADS) {
                const int s = keys[j];
                if (s < 0) continue;
                const uint4* krow = reinterpret_cast<const uint4*>(kvb + static_cast<int64_t>(s) * DQK);
                float2 acc[DISTILL_HG];
#pragma unroll
                for (int h = 0; h < DISTILL_HG; ++h) acc[h] = make_float2(0.f, 0.f);
#pragma unroll 2
                for (int c = 0; c < DQK / 8; ++c) {
                    const uint4 raw = __ldg(krow + c);
                    const float2 k0 = bf16x2_to_float2(raw.x), k1 = bf16x2_to_float2(raw.y);
                    const float2 k2 = bf16x2_to_float2(raw.z), k3 = bf16x2_to_float2(raw.w);
#pragma unroll
                    for (int h = 0; h < DISTILL_HG; ++h) {
                        if (h < hgn) {
                            const float4 qa = *reinterpret_cast<const float4*>(qf + h * DQK + c * 8);
                            const float4 qb = *reinterpret_cast<const float4*>(qf + h * DQK + c * 8 + 4);
                            acc[h] = __ffma2_rn(make_float2(qa.x, qa.y), k0, acc[h]);
                            acc[h] = __ffma2_rn(make_float2(qa.z, qa.w), k1, acc[h]);
                            acc[h] = __ffma2_rn(make_float2(qb.x, qb.y), k2, acc[h]);
                            acc[h] = __ffma2_rn(make_float2(qb.z, qb.w), k3, acc[h]);
                        }
                    }
                }
#pragma unroll
                for (int h = 0; h < DISTILL_HG; ++h) {
                    if (h < hgn) {
                        const float z = (acc[h].x + acc[h].y) * p.sm_scale;
                        zs[h * topk + j] = z;
                        ml_merge(m[h], lsum[h], z, 1.f);
                    }
                }
            }
            // per-head normaliser: warp, then block
#pragma unroll
            for (int h = 0; h < DISTILL_HG; ++h) {
                for (int o = 16; o > 0; o >>= 1) {
                    const float m2 = __shfl_xor_sync(0xffffffffu, m[h], o);
                    const float l2 = __shfl_xor_sync(0xffffffffu, lsum[h], o);
                    ml_merge(m[h], lsum[h], m2, l2);
                }
            }
            if (lane == 0) {
#pragma unroll
                for (int h = 0; h < DISTILL_HG; ++h) {
                    red_m[warp * DISTILL_HG + h] = m[h];
                    red_l[warp * DISTILL_HG + h] = lsum[h];
                }
            }
            __syncthreads();
            if (tid < hgn) {
                float mm = -INFINITY, ll = 0.f;
                for (int w = 0; w < NW; ++w) ml_merge(mm, ll, red_m[w * DISTILL_HG + tid], red_l[w * DISTILL_HG + tid]);
                head_m[tid] = mm;
                head_l[tid] = ll;
            }
            __syncthreads();
            for (int j = tid; j < topk; j += DISTILL_THREADS) {
                if (keys[j] < 0) continue;
                float acc = 0.f;
                for (int h = 0; h < hgn; ++h) acc += expf(zs[h * topk + j] - head_m[h]) / head_l[h];
                P[j] += acc * inv_norm;
            }
        }
    }

    // ---- the indexer's distribution over the same keys
    __syncthreads();
    const int d_I = p.d_I;
    for (int i = tid; i < HI * d_I; i += DISTILL_THREADS) {
        const int64_t e = row * HI * d_I + i;
        qf[i] = p.fp8 ? static_cast<float>(reinterpret_cast<const __nv_fp8_e4m3*>(p.q_I)[e])
                      : __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p.q_I)[e]);
    }
    for (int h = tid; h < HI; h += DISTILL_THREADS) {
        const int64_t e = row * HI + h;
        const float wv = p.w_is_f32 ? reinterpret_cast<const float*>(p.w)[e]
                                    : __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p.w)[e]);
        wq[h] = wv * (p.q_scale ? p.q_scale[row] : 1.f);
    }
    __syncthreads();
    float zmax = -INFINITY;
    for (int j = tid; j < topk; j += DISTILL_THREADS) {
        const int s = keys[j];
        if (s < 0) continue;
        const int64_t krow = (static_cast<int64_t>(b) * p.n_k + s) * d_I;
        float dot[HI];
#pragma unroll
        for (int h = 0; h < HI; ++h) dot[h] = 0.f;
        for (int d0 = 0; d0 < d_I; d0 += 8) {
            float kf[8];
            if (p.fp8) {
                const uint2 raw = *reinterpret_cast<const uint2*>(reinterpret_cast<const uint8_t*>(p.k_I) + krow + d0);
                const uint8_t* bytes = reinterpret_cast<const uint8_t*>(&raw);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    __nv_fp8_e4m3 v;
                    v.__x = bytes[e];
                    kf[e] = static_cast<float>(v);
                }
            } else {
                const uint4 raw = *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(p.k_I) + krow + d0);
                const float2 a = bf16x2_to_float2(raw.x), bb = bf16x2_to_float2(raw.y);
                const float2 c = bf16x2_to_float2(raw.z), dd = bf16x2_to_float2(raw.w);
                kf[0] = a.x; kf[1] = a.y; kf[2] = bb.x; kf[3] = bb.y;
                kf[4] = c.x; kf[5] = c.y; kf[6] = dd.x; kf[7] = dd.y;
            }
#pragma unroll
            for (int h = 0; h < HI; ++h) {
                const float4 qa = *reinterpret_cast<const float4*>(qf + h * d_I + d0);
                const float4 qb = *reinterpret_cast<const float4*>(qf + h * d_I + d0 + 4);
                dot[h] = fmaf(qa.x, kf[0], dot[h]);
                dot[h] = fmaf(qa.y, kf[1], dot[h]);
                dot[h] = fmaf(qa.z, kf[2], dot[h]);
                dot[h] = fmaf(qa.w, kf[3], dot[h]);
                dot[h] = fmaf(qb.x, kf[4], dot[h]);
                dot[h] = fmaf(qb.y, kf[5], dot[h]);
                dot[h] = fmaf(qb.z, kf[6], dot[h]);
                dot[h] = fmaf(qb.w, kf[7], dot[h]);
            }
        }
        float score = 0.f;
#pragma unroll
        for (int h = 0; h < HI; ++h) score = fmaf(wq[h], fmaxf(dot[h], 0.f), score);
        if (p.k_scale) score *= p.k_scale[static_cast<int64_t>(b) * p.n_k + s];
        zs[j] = score;
        zmax = fmaxf(zmax, score);
    }
    zmax = block_max(zmax, scratch);
    float esum = 0.f;
    for (int j = tid; j < topk; j += DISTILL_THREADS)
        if (keys[j] >= 0) esum += expf(zs[j] - zmax);
    esum = block_sum(esum, scratch);
    const float log_z = zmax + logf(esum);
    float part = 0.f;
    for (int j = tid; j < topk; j += DISTILL_THREADS) {
        const bool ok = keys[j] >= 0;
        const float pj = ok ? P[j] : 0.f;
        if (ok && pj > 0.f) part += pj * (logf(pj) - (zs[j] - log_z));
        if (p.target) p.target[row * topk + j] = pj;
    }
    part = block_sum(part, scratch);
    if (tid == 0) p.kl[row] = part;
    (void)warp;
}

}  // namespace ic
