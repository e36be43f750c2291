// small_kernels.cuh -- the memory-light steps around the two grouped GEMMs:
// top-k routing, the fp32 router GEMM, the dispatch bookkeeping (histogram,
// scan, stable scatter), the row gather, the tile-schedule builder, the
// deterministic combine, the fp32->bf16 finalize, and dtype casts.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "gemm_sm100.cuh"

namespace moe {

constexpr int kPermTokens = 256;  // tokens per dispatch chunk (one CTA, 8 warps)
constexpr int kPermWarps = kPermTokens / 32;

// ------------------------------------------------------------------ routing

// Router logits in fp32 for fp32 inputs: logits[t,e] = sum_h x[t,h] * w[e,h].
// One CTA per token; each warp walks experts, lanes stride over h.
__global__ void router_logits_f32_kernel(const float* __restrict__ x,
                                         const float* __restrict__ gate_w, int H, int E,
                                         float* __restrict__ logits) {
    const int t = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float* xr = x + static_cast<size_t>(t) * H;
    for (int e = warp; e < E; e += blockDim.x >> 5) {
        const float* wr = gate_w + static_cast<size_t>(e) * H;
        float acc = 0.0f;
        for (int h = lane; h < H; h += 32) acc = fmaf(xr[h], wr[h], acc);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (lane == 0) logits[static_cast<size_t>(t) * E + e] = acc;
    }
}

// Top-k routing, one warp per token (see route_one_token).
__global__ void topk_kernel(float* __restrict__ logits, int n_parts, int64_t part_stride,
                            bool keep_sum, const float* __restrict__ bias, int64_t T, int E, int k,
                            float scale, int32_t* __restrict__ idx_out,
                            float* __restrict__ w_out) {
    const int64_t t = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (t >= T) return;
    route_one_token(logits, n_parts, part_stride, keep_sum, bias, t, E, k, scale, idx_out, w_out);
}

// ------------------------------------------------------------------ router statistics

constexpr int kStatsTokensPerBlock = 64;  // 8 warps x 8 tokens

// Per-block sums of the routing probabilities p[t,e] = softmax(logits[t] + bias)
// over a fixed block of 64 tokens, in a fixed order (warp w sums its 8 tokens
// in turn, then the 8 warp sums are added in warp order); also counts the
// selected experts into `counts` (integer atomics: order-independent).
__global__ void router_prob_partial_kernel(const float* __restrict__ logits,
                                           const float* __restrict__ bias,
                                           const int32_t* __restrict__ idx, int64_t T, int E,
                                           int k, float* __restrict__ partial,
                                           int32_t* __restrict__ counts) {
    __shared__ float s_sum[8][kMaxExperts];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int kPer = kMaxExperts / 32;
    float acc[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i) acc[i] = 0.0f;
    for (int q = 0; q < kStatsTokensPerBlock / 8; ++q) {
        const int64_t t = static_cast<int64_t>(blockIdx.x) * kStatsTokensPerBlock + warp * 8 + q;
        if (t >= T) break;
        float v[kPer];
        float mx = -INFINITY;
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const int e = lane + 32 * i;
            v[i] = -INFINITY;
            if (e < E) {
                v[i] = logits[t * E + e] + (bias ? bias[e] : 0.0f);
                mx = fmaxf(mx, v[i]);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        float z = 0.0f;
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            v[i] = (lane + 32 * i < E) ? expf(v[i] - mx) : 0.0f;
            z += v[i];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
#pragma unroll
        for (int i = 0; i < kPer; ++i) acc[i] += v[i] / z;
        if (lane < k) {
            const int e = idx[t * k + lane];
            if (e >= 0 && e < E) atomicAdd(&counts[e], 1);
        }
    }
#pragma unroll
    for (int i = 0; i < kPer; ++i) s_sum[warp][lane + 32 * i] = acc[i];
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        float s = 0.0f;
#pragma unroll
        for (int w = 0; w < 8; ++w) s += s_sum[w][e];
        partial[static_cast<size_t>(blockIdx.x) * E + e] = s;
    }
}

// One CTA: P = sum of the per-block sums (in block order, fp64) / T,
// f = counts / (T k), aux = E * sum_e P_e f_e (fixed-order reduction), and the
// moving averages ema_counts = m * ema_counts + (1 - m) * counts,
// ema_total = m * ema_total + (1 - m) * T.
__global__ void router_stats_final_kernel(const float* __restrict__ partial, int nblocks,
                                          const int32_t* __restrict__ counts, int64_t T, int E,
                                          int k, float momentum, float* __restrict__ P_out,
                                          float* __restrict__ f_out, float* __restrict__ aux_out,
                                          float* ema_counts, float* ema_total) {
    __shared__ double s_prod[kMaxExperts];
    const int e = threadIdx.x;
    double prod = 0.0;
    if (e < E) {
        double sum = 0.0;
        for (int b = 0; b < nblocks; ++b) sum += partial[static_cast<size_t>(b) * E + e];
        const double P = sum / static_cast<double>(T);
        const double f = static_cast<double>(counts[e]) / (static_cast<double>(T) * k);
        P_out[e] = static_cast<float>(P);
        f_out[e] = static_cast<float>(f);
        prod = P * f;
        if (ema_counts)
            ema_counts[e] = momentum * ema_counts[e] + (1.0f - momentum) * counts[e];
    }
    s_prod[e] = prod;
    __syncthreads();
    for (int s = kMaxExperts / 2; s > 0; s >>= 1) {
        if (e < s) s_prod[e] += s_prod[e + s];
        __syncthreads();
    }
    if (e == 0) {
        *aux_out = static_cast<float>(E * s_prod[0]);
        if (ema_total) *ema_total = momentum * (*ema_total) + (1.0f - momentum) * T;
    }
}

// ------------------------------------------------------------------ dispatch

// Build, for the warp's 32 tokens, one bit mask per expert of the lanes whose
// token routes to it.  A token's k experts must be distinct; a repeat, or an
// index outside [0,E), is reported through `status` and skipped.
__device__ __forceinline__ void build_lane_masks(const int32_t* __restrict__ idx, int64_t T, int E,
                                                 int k, int64_t t, uint32_t* warp_masks,
                                                 int32_t* status) {
    const int lane = threadIdx.x & 31;
    if (t < T) {
        for (int j = 0; j < k; ++j) {
            const int e = idx[t * k + j];
            if (e < 0 || e >= E) {
                set_device_error(status, DEV_ERR_BAD_INDEX);
                continue;
            }
            const uint32_t old = atomicOr(&warp_masks[e], 1u << lane);
            if (old & (1u << lane)) set_device_error(status, DEV_ERR_BAD_INDEX);
        }
    }
}

// Pass 1: per-chunk expert histogram hist[chunk, e].
__global__ void dispatch_count_kernel(const int32_t* __restrict__ idx, int64_t T, int E, int k,
                                      int32_t* __restrict__ hist, int32_t* status) {
    __shared__ uint32_t masks[kPermWarps][kMaxExperts];
    for (int i = threadIdx.x; i < kPermWarps * kMaxExperts; i += blockDim.x)
        (&masks[0][0])[i] = 0u;
    __syncthreads();
    const int warp = threadIdx.x >> 5;
    const int64_t t = static_cast<int64_t>(blockIdx.x) * kPermTokens + threadIdx.x;
    build_lane_masks(idx, T, E, k, t, masks[warp], status);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int c = 0;
#pragma unroll
        for (int w = 0; w < kPermWarps; ++w) c += __popc(masks[w][e]);
        hist[static_cast<size_t>(blockIdx.x) * E + e] = c;
    }
}

// Exclusive prefix sum over the CTA (blockDim.x a multiple of 32, <= 1024).
// `s_warp` is 32 ints of shared scratch; every thread must call it.
__device__ __forceinline__ int block_exclusive_scan(int v, int* s_warp, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nwarps = blockDim.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) s_warp[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = lane < nwarps ? s_warp[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        s_warp[lane] = w;
    }
    __syncthreads();
    const int result = (warp > 0 ? s_warp[warp - 1] : 0) + x - v;
    if (total) *total = s_warp[nwarps - 1];
    __syncthreads();
    return result;
}

// Tile schedule entry of one segment (see SchedPtrs): chunk count and chunk
// length for rows split into chunks of at most nmax rows (multiples of 16).
__device__ __forceinline__ void segment_chunks(int rows, int nmax, int* chunks, int* chunk_len) {
    const int c = (rows + nmax - 1) / nmax;
    int cl = 16;
    if (c > 0) cl = (((rows + c - 1) / c) + 15) & ~15;
    *chunks = c;
    *chunk_len = cl;
}

// Pass 2 (one CTA of 512 threads; thread s handles expert / segment s): per-chunk
// bases, expert counts and offsets, and the tile schedules of the gate/up and
// down GEMMs (routed experts, then the shared expert as one more segment).
__global__ void __launch_bounds__(512) dispatch_scan_kernel(
    const int32_t* __restrict__ hist, int nchunks, int E, int64_t T, int k, int num_shared,
    int32_t* __restrict__ base, int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
    int32_t* sched_gu, int nmax_gu, int32_t* sched_dn, int nmax_dn) {
    __shared__ int s_warp[32];
    const int tid = threadIdx.x;
    ptx::grid_dep_wait();  // the histogram comes from the previous launch
    ptx::grid_dep_launch();
    int cnt = 0;
    if (tid < E) {
        int running = 0;
#pragma unroll 4
        for (int c = 0; c < nchunks; ++c) {
            const int v = hist[static_cast<size_t>(c) * E + tid];
            base[static_cast<size_t>(c) * E + tid] = running;
            running += v;
        }
        cnt = running;
        counts[tid] = cnt;
    }
    int total = 0;
    const int off = block_exclusive_scan(cnt, s_warp, &total);
    if (tid < E) offsets[tid] = off;
    if (tid == 0) offsets[E] = total;

    const int routed = static_cast<int>(T * k);
    const int nseg = E + (num_shared ? 1 : 0);
    int rows = 0, b0_gu = 0, b0_dn = 0, o0 = 0;
    if (tid < E) {
        rows = cnt;
        b0_gu = b0_dn = o0 = off;
    } else if (tid == E && num_shared) {
        rows = static_cast<int>(T);
        b0_gu = 0;       // gate/up: the shared expert reads x itself
        b0_dn = routed;  // down: its h rows follow the routed rows
        o0 = routed;
    }
    const bool active = tid < nseg;
    for (int which = 0; which < 2; ++which) {
        int32_t* sched = which == 0 ? sched_gu : sched_dn;
        const int nmax = which == 0 ? nmax_gu : nmax_dn;
        int chunks = 0, cl = 16;
        if (active) segment_chunks(rows, nmax, &chunks, &cl);
        int tot = 0;
        const int pre = block_exclusive_scan(chunks, s_warp, &tot);
        if (sched && active) {
            const SchedPtrs sp = sched_ptrs(sched, nseg);
            const_cast<int32_t*>(sp.prefix)[tid] = pre;
            const_cast<int32_t*>(sp.b_row0)[tid] = which == 0 ? b0_gu : b0_dn;
            const_cast<int32_t*>(sp.out_row0)[tid] = o0;
            const_cast<int32_t*>(sp.rows)[tid] = rows;
            const_cast<int32_t*>(sp.chunk_len)[tid] = cl;
            if (tid == 0) const_cast<int32_t*>(sp.prefix)[nseg] = tot;
        }
    }
}

// Pass 3: stable positions.  Row order inside an expert is (token, slot);
// a token lists an expert at most once, so ordering by token is enough.
__global__ void dispatch_scatter_kernel(const int32_t* __restrict__ idx,
                                        const float* __restrict__ topk_w, int64_t T, int E, int k,
                                        const int32_t* __restrict__ base,
                                        const int32_t* __restrict__ offsets,
                                        int32_t* __restrict__ pos, int32_t* __restrict__ src,
                                        float* __restrict__ row_w, int32_t* status) {
    __shared__ uint32_t masks[kPermWarps][kMaxExperts];
    __shared__ int32_t wbase[kPermWarps][kMaxExperts];
    for (int i = threadIdx.x; i < kPermWarps * kMaxExperts; i += blockDim.x)
        (&masks[0][0])[i] = 0u;
    ptx::grid_dep_wait();  // bases and offsets come from the previous launch
    ptx::grid_dep_launch();
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t t = static_cast<int64_t>(blockIdx.x) * kPermTokens + threadIdx.x;
    build_lane_masks(idx, T, E, k, t, masks[warp], nullptr);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int running = offsets[e] + base[static_cast<size_t>(blockIdx.x) * E + e];
#pragma unroll
        for (int w = 0; w < kPermWarps; ++w) {
            wbase[w][e] = running;
            running += __popc(masks[w][e]);
        }
    }
    __syncthreads();
    if (t < T) {
        const uint32_t lt = (1u << lane) - 1u;
        for (int j = 0; j < k; ++j) {
            const int e = idx[t * k + j];
            if (e < 0 || e >= E) continue;
            const int r = wbase[warp][e] + __popc(masks[warp][e] & lt);
            pos[t * k + j] = r;
            src[r] = static_cast<int32_t>(t);
            if (row_w) row_w[r] = topk_w[t * k + j];
        }
    }
}

// Schedule for a caller-described grouping (staged FFN entry point):
// segment g covers rows [offsets[g], offsets[g+1]) of x_perm / y_perm.
__global__ void schedule_from_offsets_kernel(const int32_t* __restrict__ offsets, int ngroups,
                                             int64_t max_rows, int32_t* sched_gu, int nmax_gu,
                                             int32_t* sched_dn, int nmax_dn, int32_t* status) {
    if (threadIdx.x != 0) return;
    const SchedPtrs sg = sched_ptrs(sched_gu, ngroups);
    const SchedPtrs sd = sched_ptrs(sched_dn, ngroups);
    int accg = 0, accd = 0;
    for (int g = 0; g < ngroups; ++g) {
        int o0 = offsets[g], o1 = offsets[g + 1];
        if (o0 < 0 || o1 < o0 || o1 > max_rows) {
            set_device_error(status, DEV_ERR_BAD_INDEX);
            o0 = 0;
            o1 = 0;
        }
        const int r = o1 - o0;
        const int cg = (r + nmax_gu - 1) / nmax_gu;
        const int cd = (r + nmax_dn - 1) / nmax_dn;
        int lg = 16, ld = 16;
        if (cg > 0) lg = (((r + cg - 1) / cg) + 15) & ~15;
        if (cd > 0) ld = (((r + cd - 1) / cd) + 15) & ~15;
        const_cast<int32_t*>(sg.prefix)[g] = accg;
        const_cast<int32_t*>(sg.b_row0)[g] = o0;
        const_cast<int32_t*>(sg.out_row0)[g] = o0;
        const_cast<int32_t*>(sg.rows)[g] = r;
        const_cast<int32_t*>(sg.chunk_len)[g] = lg;
        const_cast<int32_t*>(sd.prefix)[g] = accd;
        const_cast<int32_t*>(sd.b_row0)[g] = o0;
        const_cast<int32_t*>(sd.out_row0)[g] = o0;
        const_cast<int32_t*>(sd.rows)[g] = r;
        const_cast<int32_t*>(sd.chunk_len)[g] = ld;
        accg += cg;
        accd += cd;
    }
    const_cast<int32_t*>(sg.prefix)[ngroups] = accg;
    const_cast<int32_t*>(sd.prefix)[ngroups] = accd;
}

// ------------------------------------------------------------------ outputs

// out[t,h] = cast(acc[t,h]), 4 elements per thread.
template <typename TOut>
__global__ void finalize_kernel(const float* __restrict__ acc, TOut* __restrict__ out, int64_t n4) {
    ptx::grid_dep_wait();  // the accumulator comes from the previous launch
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const float4 v = reinterpret_cast<const float4*>(acc)[i];
        if constexpr (sizeof(TOut) == 4) {
            reinterpret_cast<float4*>(out)[i] = v;
        } else {
            __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
            __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
            uint2 p;
            p.x = *reinterpret_cast<uint32_t*>(&a);
            p.y = *reinterpret_cast<uint32_t*>(&b);
            reinterpret_cast<uint2*>(out)[i] = p;
        }
    }
}

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) {
    return v;
}
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
    return __bfloat162float(v);
}

// Deterministic combine: out[t] = sum_j w[t,j] * y_perm[pos[t,j]] (+ shared_y[t]),
// summed in slot order in fp32.  One CTA per token.
template <typename T>
__global__ void combine_kernel(const T* __restrict__ y_perm, const int32_t* __restrict__ pos,
                               const float* __restrict__ w, const T* __restrict__ shared_y,
                               int64_t T_, int H, int k, int64_t n_rows, T* __restrict__ out,
                               int32_t* status) {
    const int64_t t = blockIdx.x;
    __shared__ int32_t s_pos[kMaxExperts];
    __shared__ float s_w[kMaxExperts];
    for (int j = threadIdx.x; j < k; j += blockDim.x) {
        int p = pos[t * k + j];
        if (p < 0 || p >= n_rows) {
            set_device_error(status, DEV_ERR_BAD_INDEX);
            p = -1;
        }
        s_pos[j] = p;
        s_w[j] = w[t * k + j];
    }
    __syncthreads();
    for (int h = threadIdx.x; h < H; h += blockDim.x) {
        float acc = 0.0f;
        for (int j = 0; j < k; ++j) {
            if (s_pos[j] >= 0)
                acc = fmaf(s_w[j], to_f32(y_perm[static_cast<int64_t>(s_pos[j]) * H + h]), acc);
        }
        if (shared_y) acc += to_f32(shared_y[t * H + h]);
        if constexpr (sizeof(T) == 4) out[t * H + h] = acc;
        else out[t * H + h] = __float2bfloat16_rn(acc);
    }
}

// Fixed-order combine of weighted expert rows (the down GEMM already applied
// the routing weights): out[t] = sum_j y[pos[t,j]] (j = 0..k-1 in slot order)
// + y[shared_row0 + t] when shared_row0 >= 0, summed in fp32.  One warp per
// (token, segment of 32*kVPL 16-byte vectors of H), each lane kVPL vectors of
// each row; kBatch rows' loads are in flight before any is added (the sums
// stay in slot order), so even a few tokens spread over many warps.  y is
// bf16 (8 values per vector) or fp32 (4 values per vector).
template <typename TIn>
__device__ __forceinline__ void add_vec(float (&acc)[16 / sizeof(TIn)], const uint4& q) {
    if constexpr (sizeof(TIn) == 2) {
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(h2[e]);
            acc[2 * e] += f.x;
            acc[2 * e + 1] += f.y;
        }
    } else {
        acc[0] += __uint_as_float(q.x);
        acc[1] += __uint_as_float(q.y);
        acc[2] += __uint_as_float(q.z);
        acc[3] += __uint_as_float(q.w);
    }
}

template <typename TIn, typename TOut, int kBatch, int kVPL>
__global__ void gather_sum_kernel(const TIn* __restrict__ y, const int32_t* __restrict__ pos,
                                  int64_t T, int H, int k, int64_t n_rows, int64_t shared_row0,
                                  TOut* __restrict__ out, int32_t* status) {
    constexpr int kVE = 16 / static_cast<int>(sizeof(TIn));  // values per 16-byte vector
    constexpr int kSeg = 32 * kVPL;                           // vectors per warp segment
    const int lane = threadIdx.x & 31;
    const int nvec = H / kVE;
    const int nseg = (nvec + kSeg - 1) / kSeg;
    ptx::grid_dep_wait();  // the rows come from the previous launch
    const int64_t gw = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int64_t t = gw / nseg;
    if (t >= T) return;
    const int seg = static_cast<int>(gw - t * nseg);
    int my_pos = -1;
    if (lane < k) {
        const int p = pos[t * k + lane];
        if (p < 0 || p >= n_rows) set_device_error(status, DEV_ERR_BAD_INDEX);
        else my_pos = p;
    }
    const uint4* yv = reinterpret_cast<const uint4*>(y);
    const int64_t row_vecs = nvec;
    int vi[kVPL];
    bool ok[kVPL];
    float acc[kVPL][kVE];
#pragma unroll
    for (int u = 0; u < kVPL; ++u) {
        vi[u] = seg * kSeg + 32 * u + lane;
        ok[u] = vi[u] < nvec;
#pragma unroll
        for (int e = 0; e < kVE; ++e) acc[u][e] = 0.0f;
    }
    // rows in slot order (the shared expert's last)
    const int n_rows_t = k + (shared_row0 >= 0 ? 1 : 0);
    for (int j0 = 0; j0 < n_rows_t; j0 += kBatch) {
        uint4 q[kBatch][kVPL];
        bool has[kBatch];
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            const int j = j0 + b;
            int64_t r = -1;
            if (j < k) r = __shfl_sync(0xffffffffu, my_pos, j & 31);
            else if (j < n_rows_t) r = shared_row0 + t;
            has[b] = r >= 0;
#pragma unroll
            for (int u = 0; u < kVPL; ++u)
                if (has[b] && ok[u]) q[b][u] = yv[r * row_vecs + vi[u]];
        }
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
#pragma unroll
            for (int u = 0; u < kVPL; ++u)
                if (has[b] && ok[u]) add_vec<TIn>(acc[u], q[b][u]);
        }
    }
#pragma unroll
    for (int u = 0; u < kVPL; ++u) {
        if (!ok[u]) continue;
        TOut* o = out + t * H + static_cast<int64_t>(vi[u]) * kVE;
        if constexpr (sizeof(TOut) == 2 && kVE == 8) {
            uint4 qo;
            __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(&qo);
#pragma unroll
            for (int e = 0; e < 4; ++e) h2[e] = __floats2bfloat162_rn(acc[u][2 * e], acc[u][2 * e + 1]);
            *reinterpret_cast<uint4*>(o) = qo;
        } else if constexpr (sizeof(TOut) == 2) {
            uint2 qo;
            __nv_bfloat162* h2 = reinterpret_cast<__nv_bfloat162*>(&qo);
            h2[0] = __floats2bfloat162_rn(acc[u][0], acc[u][1]);
            h2[1] = __floats2bfloat162_rn(acc[u][2], acc[u][3]);
            *reinterpret_cast<uint2*>(o) = qo;
        } else {
#pragma unroll
            for (int e = 0; e < kVE; e += 4)
                *reinterpret_cast<float4*>(o + e) =
                    make_float4(acc[u][e], acc[u][e + 1], acc[u][e + 2], acc[u][e + 3]);
        }
    }
}

// ------------------------------------------------------------------ wait self-check

// One thread runs the two bounded waits the kernels rely on against events
// that never happen: an mbarrier nobody arrives on and a global counter nobody
// increments.  Each gives up after limit_cycles and records MOE_ERR_TIMEOUT in
// the error word; `result` gets one bit per wait that (correctly) gave up.
__global__ void wait_selftest_kernel(const int32_t* counter, uint64_t limit_cycles,
                                     int32_t* status, int32_t* result) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0) return;
    ptx::mbar_init(&bar, 1);
    ptx::fence_mbar_init();
    int bits = 0;
    if (!ptx::mbar_wait(&bar, 0, nullptr, limit_cycles)) {
        set_device_error(status, DEV_ERR_TIMEOUT);
        bits |= 1;
    }
    if (!ptx::wait_counter_at_least(counter, 1, limit_cycles)) {
        set_device_error(status, DEV_ERR_TIMEOUT);
        bits |= 2;
    }
    *result = bits;
}

// ------------------------------------------------------------------ FP8 (E4M3) quantization
//
// Scales are powers of two, s = 2^n with n the smallest integer such that
// 448 * 2^n >= amax (448 is the largest E4M3 value; s = 1 when amax == 0), so
// v / s is exact and the E4M3 code of v / s does not depend on the precision
// the division is done in.

__device__ __forceinline__ float pow2_scale_f(float amax) {
    if (!(amax > 0.0f)) return 1.0f;
    int n = ilogbf(amax) - 8;  // 2^8 < 448 < 2^9
    while (ldexpf(448.0f, n) < amax) ++n;
    while (n > -126 && ldexpf(448.0f, n - 1) >= amax) --n;
    return ldexpf(1.0f, n);
}

template <typename T>
__device__ __forceinline__ float load_f32(const T* p, int64_t i);
template <>
__device__ __forceinline__ float load_f32<float>(const float* p, int64_t i) {
    return p[i];
}
template <>
__device__ __forceinline__ float load_f32<__nv_bfloat16>(const __nv_bfloat16* p, int64_t i) {
    return __bfloat162float(p[i]);
}

// Per-row quantization: for each of n_rows rows of length len (one warp per
// row), scale = pow2_scale(max |row|), codes = e4m3(row / scale).
// Row r of the output is row (r / group) * src_group_stride + r % group of the
// input (group = src_group_stride: plain rows; group = 2*I, stride 3*I: the
// gate and up rows of [E,3,I,H] expert weights); codes keep the input's layout.
// len is a multiple of 128 (so rows are 16-byte aligned): each lane reads
// 16-byte vectors (8 bf16 or 4 fp32 values), eight in flight, and writes each
// vector's codes at once.
template <typename T>
__device__ __forceinline__ void unpack_vec(const uint4& q, float (&f)[16 / sizeof(T)]) {
    if constexpr (sizeof(T) == 2) {
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&q);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 v = __bfloat1622float2(h2[e]);
            f[2 * e] = v.x;
            f[2 * e + 1] = v.y;
        }
    } else {
        f[0] = __uint_as_float(q.x);
        f[1] = __uint_as_float(q.y);
        f[2] = __uint_as_float(q.z);
        f[3] = __uint_as_float(q.w);
    }
}

template <typename T>
__global__ void quantize_rows_e4m3_kernel(const T* __restrict__ in, int64_t n_rows, int len,
                                          int64_t group, int64_t src_group_stride,
                                          uint8_t* __restrict__ q, float* __restrict__ scale) {
    constexpr int kVE = 16 / static_cast<int>(sizeof(T));  // values per 16-byte vector
    const int lane = threadIdx.x & 31;
    const int64_t r = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (r >= n_rows) return;
    const int64_t src_row = (r / group) * src_group_stride + r % group;
    const uint4* row = reinterpret_cast<const uint4*>(in + src_row * len);
    const int nv = len / kVE;
    constexpr int kU = 8;  // vectors per lane in flight before any is used
    float amax = 0.0f;
    for (int v0 = lane; v0 < nv; v0 += 32 * kU) {
        uint4 qv[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u)
            if (v0 + 32 * u < nv) qv[u] = row[v0 + 32 * u];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            if (v0 + 32 * u < nv) {
                float f[kVE];
                unpack_vec<T>(qv[u], f);
#pragma unroll
                for (int e = 0; e < kVE; ++e) amax = fmaxf(amax, fabsf(f[e]));
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float sc = pow2_scale_f(amax);
    const float inv = 1.0f / sc;  // exact: power of two
    uint8_t* qr = q + src_row * len;
    for (int v0 = lane; v0 < nv; v0 += 32 * kU) {
        uint4 qv[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u)
            if (v0 + 32 * u < nv) qv[u] = row[v0 + 32 * u];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int v = v0 + 32 * u;
            if (v < nv) {
                float f[kVE];
                unpack_vec<T>(qv[u], f);
                uint32_t c[kVE / 4];
#pragma unroll
                for (int w = 0; w < kVE / 4; ++w)
                    c[w] = static_cast<uint32_t>(ptx::e4m3x2(f[4 * w] * inv, f[4 * w + 1] * inv)) |
                           (static_cast<uint32_t>(
                                ptx::e4m3x2(f[4 * w + 2] * inv, f[4 * w + 3] * inv))
                            << 16);
                if constexpr (kVE == 8)
                    *reinterpret_cast<uint2*>(qr + static_cast<int64_t>(v) * kVE) =
                        make_uint2(c[0], c[1]);
                else
                    *reinterpret_cast<uint32_t*>(qr + static_cast<int64_t>(v) * kVE) = c[0];
            }
        }
    }
    if (lane == 0) scale[r] = sc;
}

// Per-column quantization of [n_mats][rows][cols] matrices: each thread owns
// one column of one matrix: scale = pow2_scale(max |column|).
template <typename T>
__global__ void quantize_cols_e4m3_kernel(const T* __restrict__ in, int64_t mat_stride,
                                          int64_t out_mat_stride, int n_mats, int rows, int cols,
                                          uint8_t* __restrict__ q, float* __restrict__ scale) {
    const int64_t id = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (id >= static_cast<int64_t>(n_mats) * cols) return;
    const int mat = static_cast<int>(id / cols);
    const int c = static_cast<int>(id - static_cast<int64_t>(mat) * cols);
    const T* base = in + mat * mat_stride + c;
    float amax = 0.0f;
    for (int r = 0; r < rows; ++r) amax = fmaxf(amax, fabsf(load_f32(base, static_cast<int64_t>(r) * cols)));
    const float sc = pow2_scale_f(amax);
    const float inv = 1.0f / sc;
    uint8_t* qb = q + mat * out_mat_stride + c;
    for (int r = 0; r < rows; ++r)
        qb[static_cast<int64_t>(r) * cols] =
            static_cast<uint8_t>(ptx::e4m3x2(load_f32(base, static_cast<int64_t>(r) * cols) * inv,
                                             0.0f) & 0xFF);
    scale[id] = sc;
}


}  // namespace moe
