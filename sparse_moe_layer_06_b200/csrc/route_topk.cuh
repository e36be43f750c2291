// route_topk.cuh -- routing of one token by one warp: the router logits
// (optionally the sum of a K-split GEMM's partial slices) -> softmax -> top-k
// -> renormalise -> scale.  Used by the top-k kernel and by the fused routing
// phase of the router GEMM.
#pragma once

#include <cstdint>

namespace moe {

constexpr int kMaxExperts = 256;

// Softmax -> top-k -> renormalise -> scale for token t, by the calling warp
// (all 32 lanes).  Selection runs on the fp32 logits (softmax is monotone, so
// the selected set is the top-k of the probabilities); exact ties go to the
// lower expert index.  The renormalised weights are computed as the softmax
// over the k selected logits, which equals p_j / sum_sel p (the full-softmax
// normaliser cancels).  n_parts > 1: the logits are the sum, in slice order,
// of n_parts [T,E] slices part_stride floats apart, left in the first slice
// when keep_sum is set.  Loads bypass L1 (other CTAs may have written them).
__device__ __forceinline__ void route_one_token(float* __restrict__ logits, int n_parts,
                                                int64_t part_stride, bool keep_sum,
                                                const float* __restrict__ bias, int64_t t, int E,
                                                int k, float scale, int32_t* __restrict__ idx_out,
                                                float* __restrict__ w_out) {
    const int lane = threadIdx.x & 31;
    constexpr int kPer = kMaxExperts / 32;
    float v[kPer];
    uint32_t taken = 0;
    // partial sums of a K-split GEMM, added in slice order; all loads are
    // issued before anything is stored, so they overlap
    const float* row = logits + t * E;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int e = lane + 32 * i;
        v[i] = e < E ? __ldcg(row + e) : 0.0f;
    }
    // up to kMaxParts slices: every load issued before the first addition
    constexpr int kMaxParts = 8;
    float pv[kMaxParts - 1][kPer];
#pragma unroll
    for (int q = 1; q < kMaxParts; ++q) {
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const int e = lane + 32 * i;
            pv[q - 1][i] = (q < n_parts && e < E) ? __ldcg(row + q * part_stride + e) : 0.0f;
        }
    }
#pragma unroll
    for (int q = 1; q < kMaxParts; ++q) {
        if (q < n_parts) {
#pragma unroll
            for (int i = 0; i < kPer; ++i) v[i] += pv[q - 1][i];
        }
    }
#pragma unroll 1
    for (int q = kMaxParts; q < n_parts; ++q) {
        const float* part = row + q * part_stride;
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const int e = lane + 32 * i;
            if (e < E) v[i] += __ldcg(part + e);
        }
    }
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int e = lane + 32 * i;
        if (e < E) {
            // the summed logits kept in the first slice for later readers
            if (n_parts > 1 && keep_sum) logits[t * E + e] = v[i];
            if (bias) v[i] += bias[e];
        } else {
            taken |= 1u << i;
        }
    }
    float sel_l = 0.0f, top_l = 0.0f;
    int sel_e = 0;
    float my_l = 0.0f;
    int my_e = -1;
    for (int j = 0; j < k; ++j) {
        float best = 0.0f;
        int be = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            if (!(taken & (1u << i))) {
                const int e = lane + 32 * i;
                if (be == 0x7fffffff || v[i] > best) {
                    best = v[i];
                    be = e;
                }
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const float ob = __shfl_xor_sync(0xffffffffu, best, o);
            const int oe = __shfl_xor_sync(0xffffffffu, be, o);
            const bool take = (be == 0x7fffffff) ||
                              (oe != 0x7fffffff && (ob > best || (ob == best && oe < be)));
            if (take) {
                best = ob;
                be = oe;
            }
        }
        sel_l = best;
        sel_e = be;
        if ((sel_e & 31) == lane) taken |= 1u << (sel_e >> 5);
        if (j == 0) top_l = sel_l;
        if (lane == j) {
            my_l = sel_l;
            my_e = sel_e;
        }
    }
    // weights: softmax over the k selected logits (lanes 0..k-1 hold them)
    const float ex = (lane < k) ? expf(my_l - top_l) : 0.0f;
    float sum = ex;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane < k) {
        idx_out[t * k + lane] = my_e;
        w_out[t * k + lane] = scale * (ex / sum);
    }
}

}  // namespace moe
