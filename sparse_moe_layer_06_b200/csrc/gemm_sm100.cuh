// gemm_sm100.cuh -- persistent, warp-specialised grouped GEMM on tcgen05/TMEM.
//
// One kernel template serves every contraction of the layer:
//   EPI_LOGITS      router logits      D[e, tok]  = Wgate[e,:]   . x[tok,:]
//   EPI_SWIGLU      expert gate/up     G[i, row]  = Wg_e[i,:]    . x_perm[row,:]
//                                      U[i, row]  = Wu_e[i,:]    . x_perm[row,:]
//                                      h[row, i]  = silu(clamp(G)) * clamp(U)
//   EPI_DOWN_ATOMIC expert down+combine y[h, row] = sum_i Wd_e[i,h] * h_perm[row,i]
//                                      out_acc[token(row), h] += w(row) * y
//   EPI_DOWN_STORE  expert down        y_perm[row, h] = w(row) * y  (w = 1 when no
//                                      routing weights are given)
//
// The weight matrix is always the MMA "A" operand (M = 128 weight rows per
// tile) and the token rows are the "B" operand (N = 16..NMAX rows per tile,
// any multiple of 16).  Putting tokens on N lets one kernel cover a decode
// batch (a couple of rows per expert: N = 16) and a prefill batch (hundreds of
// rows per expert: N up to 256) without padding every expert to 128 rows.
//
// Roles (320 threads = 10 warps, one CTA per SM, persistent over tiles):
//   warp 0      TMA producer: fills a STAGES-deep shared-memory ring
//   warp 1      TMEM owner + MMA issuer (one thread issues tcgen05.mma)
//   warps 2..9  epilogue: tcgen05.ld the fp32 accumulator, apply the epilogue,
//               store to global memory.  A warp may only read the 32-lane TMEM
//               quarter (warp % 4); two warps share each quarter and take
//               alternate 16-column chunks, so every scheduler has two
//               independent epilogue instruction streams to interleave.
// The accumulator is double-buffered in TMEM when it fits, so the epilogue of
// tile i overlaps the main loop of tile i+1.
//
// Variants: FP8 (E4M3 operands, tcgen05.mma kind::f8f6f4, 128 K-values per
// 128-byte row, scales applied in the epilogues); PAIR (two CTAs of a cluster
// share a tile through cta_group::2 MMAs of M = 256, each holding its own
// weight rows and half of the token rows); EPI_LOGITS with k_splits (the K
// range split over several tiles into fp32 partial slices) and, optionally,
// the routing of each token chunk once its parts are complete (route_idx).
//
// Operand layouts in shared memory (128-byte swizzle, 1024-byte atoms):
//   K-major (x, h, gate/up weights): a tile row = 64 bf16 of K = 128 bytes;
//     8 rows per atom; descriptor SBO = 1024 B; +32 B per K=16 step.
//   MN-major (down weights, stored [I,H] with H contiguous): each TMA box is
//     64 K-rows x 64 H-values (128 bytes); two boxes side by side in H make
//     the 128-wide M tile; descriptor LBO = 8192 B (between the two 64-wide H
//     halves), SBO = 1024 B (between 8-row K groups); +2048 B per K=16 step.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"
#include "route_topk.cuh"

namespace moe {

enum EpiKind : int { EPI_LOGITS = 0, EPI_SWIGLU = 1, EPI_DOWN_ATOMIC = 2, EPI_DOWN_STORE = 3 };

enum DeviceError : int { DEV_OK = 0, DEV_ERR_TIMEOUT = 5, DEV_ERR_BAD_INDEX = 6 };

__device__ __forceinline__ void set_device_error(int32_t* status, int code) {
    if (status) atomicCAS(status, 0, code);
}

// Device-built tile schedule for nseg segments (a segment = the rows that
// share one weight matrix).  int32 array of 5*(nseg+1) entries:
//   prefix[nseg+1]  exclusive prefix sum of per-segment chunk counts
//   b_row0[nseg]    first row of the segment in its B tensor map
//   out_row0[nseg]  first row of the segment in the output row space
//   rows[nseg]      rows in the segment
//   chunk_len[nseg] rows per chunk (multiple of 16, <= NMAX)
// Tiles are ordered (segment, chunk, weight block) with the weight block
// fastest, so the CTAs working at the same time share one chunk of token rows
// and, across neighbouring chunks, the same weight blocks through L2.
struct SchedPtrs {
    const int32_t* prefix;
    const int32_t* b_row0;
    const int32_t* out_row0;
    const int32_t* rows;
    const int32_t* chunk_len;
};

__host__ __device__ inline SchedPtrs sched_ptrs(const int32_t* base, int nseg) {
    SchedPtrs p;
    p.prefix = base;
    p.b_row0 = base + (nseg + 1);
    p.out_row0 = base + 2 * (nseg + 1);
    p.rows = base + 3 * (nseg + 1);
    p.chunk_len = base + 4 * (nseg + 1);
    return p;
}

constexpr int kMaxSegments = 257;  // 256 routed experts + 1 shared expert

// Token rows are fetched with TMA boxes of 16 << j rows (j = 0..4): a tile of
// n rows (a multiple of 16) takes one box per set bit of n/16, so a typical
// prefill tile needs one or two bulk copies per pipeline stage instead of n/16.
constexpr int kNumBoxSizes = 5;

struct GemmArgs {
    // A (weights).  EPI_SWIGLU: 3D map {H, I, matrices} with a {64, 128, 2} box
    // (gate and up tiles of one expert in one copy); EPI_DOWN_*: 3D map
    // {64, rows, H/64} of the [rows, H] view (strides H*2 and 128 bytes) with a
    // {64, 64, 2*MB} box; EPI_LOGITS: 2D {64, 128*MB}.
    CUtensorMap tmA0;                // ordinary segments
    CUtensorMap tmA1;                // the special segment (shared expert)
    CUtensorMap tmB0[kNumBoxSizes];  // B (token rows), box {64, 16 << j}
    CUtensorMap tmB1[kNumBoxSizes];  // B for the special segment
    const int32_t* sched;  // device schedule, or nullptr for one host-described segment
    int32_t single_rows;       // sched == nullptr: rows of the only segment
    int32_t single_chunk_len;  // sched == nullptr: rows per chunk
    int32_t nseg;
    int32_t special_seg;   // segment that uses tmA1/tmB1, or -1
    int32_t K;             // contraction length, multiple of 64
    int32_t M_total;       // valid A rows per matrix (E, I or H)
    int32_t a_seg_stride;  // A rows (EPI_SWIGLU: matrices) between segments in tmA0
    int32_t a_off0;        // A row (EPI_SWIGLU: matrix) offset of the first matrix
    int32_t a_off1;        // unused (kept zero)
    void* out;
    int32_t out_ld;
    int32_t n_tokens;          // EPI_DOWN_ATOMIC: rows of the accumulator;
                               // EPI_SWIGLU row gather: rows of gather_src
    const int32_t* row_token;  // EPI_DOWN_ATOMIC: token of each routed row
    const float* row_weight;   // EPI_DOWN_ATOMIC: routing weight of each routed row
    int32_t routed_rows;       // rows >= routed_rows belong to the shared expert
    float clip;                // EPI_SWIGLU clamp limit (+inf: none)
    int32_t out_f32;           // EPI_DOWN_STORE: fp32 (1) or bf16 (0) output
    int32_t l2_hints;          // 1: weights evict-first, token rows evict-last; 0: none
    // EPI_LOGITS: the K range split into k_splits parts (>= 1, <= K / 64), one
    // tile each; part s writes its partial sums at out + s * split_stride
    int32_t k_splits;
    int64_t split_stride;
    // EPI_LOGITS, fused routing (route_idx set; one tile per CTA, all CTAs
    // resident: a cooperative launch): after writing its partial logits each
    // CTA counts itself in on route_count[chunk], waits (bounded) until all
    // k_splits parts of its token chunk are written, and then routes its share
    // of the chunk's tokens (softmax, top-k, renormalised weights x scale)
    int32_t* route_idx;
    float* route_w;
    const float* route_bias;
    int32_t* route_count;
    int32_t route_k;
    float route_scale;
    int32_t route_keep_sum;
    // EPI_SWIGLU row gather: when gather_tok != nullptr, ordinary segments
    // take their token rows straight from gather_src ([n_tokens, K] bf16, or
    // E4M3 codes in the gather-warp kernels) at
    // rows gather_tok[b_row + i] instead of from tmB0 (the permuted copy)
    const int32_t* gather_tok;
    const void* gather_src;
    // FP8 (E4M3) operands: per weight-channel scales (EPI_SWIGLU: gate then up
    // row scales, 2*M_total per segment; EPI_DOWN_*: column scales, M_total per
    // segment), the shared expert's scales, per-token scales of the token rows
    // (EPI_SWIGLU) and the fixed scale of h (EPI_DOWN_*)
    const float* scale_w;
    const float* scale_w_special;
    const float* token_scale;
    float h_scale;      // a power of two
    float h_scale_inv;  // its exact reciprocal
    int32_t* status;           // device error word
    // K order: 0 = every tile runs K from its first step; 1 = each tile starts
    // at a tile-dependent step and wraps around (the sum order of a tile is
    // still fixed), so CTAs running together read different K bands of the
    // weights instead of the same one in lockstep
    int32_t k_rotate;
    // Programmatic dependent launch: every thread that reads an earlier
    // launch's output waits for it first (griddepcontrol.wait).  With
    // pdl_trigger_early the next launch may start as soon as this grid has
    // passed that wait (otherwise when each CTA has issued all its copies).
    int32_t pdl_trigger_early;
    // L2 policy of the weights of a segment cut into several token chunks:
    // 0 evict-first (like a single-chunk segment), 1 normal, 2 evict-last.
    // Every chunk of such a segment reads the same weight tiles, and the
    // chunks run at about the same time, so keeping the tiles in L2 turns the
    // later chunks' weight reads into L2 hits.
    int32_t multi_chunk_policy;
};

// Compile-time shape of one instantiation.
//   NMAX  largest token-row tile (MMA N), a multiple of 16 in [16, 256]
//   MB    128-row weight sub-tiles per tile: the gate and the up matrix for
//         EPI_SWIGLU (MB = 2), else 1 or 2 adjacent 128-row blocks of one
//         matrix (two MMAs sharing each token tile)
// The pipeline depth is whatever fits the 227 KB of shared memory.
//   ET    operand element type: 0 bf16 (kind::f16), 1 E4M3 (kind::f8f6f4:
//         128 K-elements per 128-byte row per stage instead of 64, scales
//         applied in the epilogue), 2 fp32 read as TF32 (kind::tf32: 32
//         K-elements per 128-byte row; h and the output rows stay fp32)
template <int EPI, int NMAX, int MB, int ET = 0, bool PAIR = false, int GW = 0>
struct GemmCfg {
    static_assert(NMAX % 16 == 0 && NMAX >= 16 && NMAX <= 256, "N tile");
    static_assert(MB == 1 || MB == 2, "weight sub-tiles");
    static_assert(EPI != EPI_SWIGLU || MB == 2, "gate/up needs both matrices");
    static constexpr bool kSwiGLU = (EPI == EPI_SWIGLU);
    static constexpr bool kDown = (EPI == EPI_DOWN_ATOMIC || EPI == EPI_DOWN_STORE);
    static constexpr int kNumA = MB;
    static_assert(ET >= 0 && ET <= 2, "element type");
    static constexpr bool kFP8 = (ET == 1);
    static constexpr bool kTF32 = (ET == 2);
    static constexpr int kElemBytes = kFP8 ? 1 : (kTF32 ? 4 : 2);
    static constexpr int kKStep = 128 / kElemBytes;  // K elements per stage (128-byte rows)
    static constexpr int kATileBytes = 128 * 128;  // 128 rows x 64 bf16
    static constexpr int kABytes = kNumA * kATileBytes;
    // PAIR: the two CTAs of a cluster run one tile with cta_group::2 MMAs of
    // M = 256 (each CTA its 128 weight rows of every sub-tile) and each CTA
    // holds half of the NMAX token rows
    static_assert(!PAIR || (NMAX % 32 == 0 && EPI != EPI_LOGITS), "pair tile");
    static constexpr int kBRows = PAIR ? NMAX / 2 : NMAX;
    static constexpr int kBBytes = kBRows * 128;  // token rows x 128 bytes
    static constexpr int kStageBytes = kABytes + kBBytes;
    static_assert(kStageBytes % 1024 == 0, "stage alignment");
    static constexpr int kAccCols = kNumA * NMAX;  // sub-tile j at column j*NMAX
    static constexpr int kAccStages = (2 * kAccCols <= 512) ? 2 : 1;
    static constexpr int kTmemNeed = kAccStages * kAccCols;
    static constexpr int kTmemCols = kTmemNeed <= 32    ? 32
                                     : kTmemNeed <= 64  ? 64
                                     : kTmemNeed <= 128 ? 128
                                     : kTmemNeed <= 256 ? 256
                                                        : 512;
    static_assert(kTmemNeed <= 512, "TMEM columns");
    // tail: 1 KB alignment slack + barriers/flags + the schedule (5 arrays)
    // + (EPI_DOWN_ATOMIC) two buffers of the token and weight of each column
    static constexpr int kBarrierBytes = 512;
    // (rounded to 128 bytes so that what follows stays 128-byte aligned)
    static constexpr int kSchedBytes = (5 * (kMaxSegments + 1) * 4 + 127) / 128 * 128;
    static constexpr bool kMeta = kDown || (kSwiGLU && kFP8);  // per-column metadata
    static constexpr int kMetaBytes = kMeta ? 2 * NMAX * 8 : 0;
    static constexpr int kEpiWarps = 8;
    // EPI_SWIGLU: token index of each row of the current tile (row gather)
    static constexpr int kGatherBytes = kSwiGLU ? NMAX * 8 : 0;
    static constexpr int kTailBytes =
        1024 + kBarrierBytes + kSchedBytes + kMetaBytes + kGatherBytes;
    static constexpr int kMaxSmem = 227 * 1024;
    static constexpr int kStagesRaw = (kMaxSmem - kTailBytes) / kStageBytes;
    static constexpr int kStages = kStagesRaw > 12 ? 12 : kStagesRaw;
    static_assert(kStages >= 2, "pipeline depth");
    static constexpr int kSmemBytes = kStages * kStageBytes + kTailBytes;
    // barrier area: full/empty per stage, accumulator full/empty x2, final,
    // metadata x2 (8 bytes each), then the TMEM slot and two flags
    static_assert((2 * kStages + 7) * 8 + 3 * 4 <= kBarrierBytes, "barrier area");
    // GW > 0 (EPI_SWIGLU with the row gather): that many more warps copy the
    // gathered token rows; the producer warp then only issues the weight copies
    static_assert(GW == 0 || (EPI == EPI_SWIGLU && ET != 2 && !PAIR), "gather warps");
    static constexpr int kThreads = 32 * (2 + kEpiWarps + GW);
};

struct TileInfo {
    int seg, blk, chunk;
    int b_row, out_row;
    int n_valid, n_mma;
    bool special;
};

// Shared-memory copy of the schedule (same layout as SchedPtrs, nseg+1 stride).
struct SmemSched {
    int32_t* prefix;
    int32_t* b_row0;
    int32_t* out_row0;
    int32_t* rows;
    int32_t* chunk_len;
};

__device__ __forceinline__ bool decode_tile(int t, int nblk, int nseg, const SmemSched& ss,
                                            int special_seg, TileInfo& ti) {
    int lo = 0, hi = nseg;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (ss.prefix[mid] * nblk <= t) lo = mid;
        else hi = mid;
    }
    const int local = t - ss.prefix[lo] * nblk;
    ti.seg = lo;
    ti.chunk = local / nblk;
    ti.blk = local - ti.chunk * nblk;
    const int cl = ss.chunk_len[lo];
    const int first = ti.chunk * cl;
    int n = ss.rows[lo] - first;
    if (n > cl) n = cl;
    ti.n_valid = n;
    ti.n_mma = (n + 15) & ~15;
    ti.b_row = ss.b_row0[lo] + first;
    ti.out_row = ss.out_row0[lo] + first;
    ti.special = (lo == special_seg);
    return n > 0;
}

// First K step (relative to the tile's range of `span` steps) of a tile whose
// K loop is rotated: spread over the range by weight block, shifted by
// segment and chunk, so that concurrently running tiles (consecutive weight
// blocks of a few segments) start at different K offsets.
__device__ __forceinline__ int k_rotation(const TileInfo& ti, int span, int nblk) {
    if (span <= 1) return 0;
    return (ti.blk * span / nblk + ti.seg * 7 + ti.chunk * 3) % span;
}

// Reciprocal of d >= 1 with the hardware approximation (relative error ~2^-23;
// 1/inf = 0, the correct limit of the SiLU gate).
__device__ __forceinline__ float fast_rcp(float d) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(d));
    return r;
}

using bf16_raw_ptr = const __nv_bfloat16*;

__device__ __forceinline__ float clamp_keep_nan(float v, float lim) {
    return v > lim ? lim : (v < -lim ? -lim : v);
}

// Output rows from the accumulator layout (one output column m per lane, 16
// token rows per chunk): the lanes of a pair (m even, m + 1) store 2-element
// units, the even lane those of the even token rows, the odd lane those of the
// odd ones.  One shuffle carries two bf16 (or four E4M3) values, so a chunk
// of 16 token rows takes 4 (2) shuffles and 8 stores per lane.  Each value is
// rounded on its own, as a single conversion would round it.
__device__ __forceinline__ uint32_t bf16x2_bits(float lo, float hi) {
    const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&p);
}

// bf16 rows: a[j] is this lane's value for token row j of the chunk; row j
// starts at element `row0 + j * ld` (row0 = the chunk's first row at the even
// lane's column).  ok(j): whether token row j is stored.
template <typename OkFn>
__device__ __forceinline__ void store_pairs_bf16(__nv_bfloat16* out, size_t row0, size_t ld,
                                                 const float (&a)[16], bool odd, OkFn ok) {
#pragma unroll
    for (int j = 0; j < 16; j += 4) {
        const uint32_t own = bf16x2_bits(odd ? a[j + 1] : a[j], odd ? a[j + 3] : a[j + 2]);
        const uint32_t snd = bf16x2_bits(odd ? a[j] : a[j + 1], odd ? a[j + 2] : a[j + 3]);
        const uint32_t rcv = __shfl_xor_sync(0xffffffffu, snd, 1);
        const uint32_t ev = odd ? rcv : own;  // the even lane's values of the two rows
        const uint32_t od = odd ? own : rcv;  // the odd lane's
        const int r = j + (odd ? 1 : 0);
        if (ok(r))
            *reinterpret_cast<uint32_t*>(out + row0 + r * ld) = __byte_perm(ev, od, 0x5410);
        if (ok(r + 2))
            *reinterpret_cast<uint32_t*>(out + row0 + (r + 2) * ld) = __byte_perm(ev, od, 0x7632);
    }
}

// E4M3 rows, as store_pairs_bf16 (byte offsets).
template <typename OkFn>
__device__ __forceinline__ void store_pairs_e4m3(uint8_t* out, size_t row0, size_t ld,
                                                 const float (&a)[16], bool odd, OkFn ok) {
#pragma unroll
    for (int j = 0; j < 16; j += 8) {
        uint32_t own = 0, snd = 0;
#pragma unroll
        for (int g = 0; g < 2; ++g) {
            const int b = j + 4 * g;
            own |= static_cast<uint32_t>(ptx::e4m3x2(odd ? a[b + 1] : a[b], odd ? a[b + 3] : a[b + 2]))
                   << (16 * g);
            snd |= static_cast<uint32_t>(ptx::e4m3x2(odd ? a[b] : a[b + 1], odd ? a[b + 2] : a[b + 3]))
                   << (16 * g);
        }
        const uint32_t rcv = __shfl_xor_sync(0xffffffffu, snd, 1);
        const uint32_t ev = odd ? rcv : own;
        const uint32_t od = odd ? own : rcv;
        const int r = j + (odd ? 1 : 0);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            // byte q of each lane's word: token row r + 2q
            if (ok(r + 2 * q))
                *reinterpret_cast<uint16_t*>(out + row0 + (r + 2 * q) * ld) =
                    static_cast<uint16_t>(__byte_perm(ev, od, q | ((4 + q) << 4)));
        }
    }
}

template <int EPI, int NMAX, int MB, int ET, bool PAIR, int GW>
__global__ void __launch_bounds__(GemmCfg<EPI, NMAX, MB, ET, PAIR, GW>::kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ GemmArgs args) {
    using C = GemmCfg<EPI, NMAX, MB, ET, PAIR, GW>;
    constexpr bool FP8 = C::kFP8;
    constexpr bool TF32 = C::kTF32;
    constexpr int CG = PAIR ? 2 : 1;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte aligned ring (the 128-byte swizzle atoms need it)
    uint8_t* ring = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t* tail = ring + C::kStages * C::kStageBytes;
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(tail);
    uint64_t* empty_bar = full_bar + C::kStages;
    uint64_t* accf_bar = empty_bar + C::kStages;
    uint64_t* acce_bar = accf_bar + 2;
    uint64_t* final_bar = acce_bar + 2;
    uint64_t* metaf_bar = final_bar + 1;  // EPI_DOWN_ATOMIC column metadata ready (x2)
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(metaf_bar + 2);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    volatile int* route_go = abort_flag + 1;  // EPI_LOGITS fused routing: the chunk is complete
    int32_t* s_sched = reinterpret_cast<int32_t*>(tail + C::kBarrierBytes);
    uint8_t* s_meta = tail + C::kBarrierBytes + C::kSchedBytes;
    // gathered tile: element offset of each row's token in the source
    int64_t* s_goff = reinterpret_cast<int64_t*>(s_meta + C::kMetaBytes);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int nseg = args.sched ? args.nseg : 1;
    // PAIR: rank 0 of the cluster (the leader) issues the MMAs for both CTAs;
    // both walk the same tile sequence, one cluster per unit of the grid
    const uint32_t rank = PAIR ? ptx::cluster_ctarank() : 0u;
    const int unit = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
    const int units = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
    SmemSched ss;
    ss.prefix = s_sched;
    ss.b_row0 = s_sched + (nseg + 1);
    ss.out_row0 = s_sched + 2 * (nseg + 1);
    ss.rows = s_sched + 3 * (nseg + 1);
    ss.chunk_len = s_sched + 4 * (nseg + 1);
    if (args.sched) {
        for (int i = threadIdx.x; i < 5 * (nseg + 1); i += blockDim.x)
            s_sched[i] = __ldcg(args.sched + i);  // (L2: written by an earlier launch)
    } else if (threadIdx.x == 0) {
        const int cl = args.single_chunk_len;
        ss.prefix[0] = 0;
        ss.prefix[1] = (args.single_rows + cl - 1) / cl;
        ss.b_row0[0] = 0;
        ss.out_row0[0] = 0;
        ss.rows[0] = args.single_rows;
        ss.chunk_len[0] = cl;
    }
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            // GW > 0: one arrival of every gather lane per stage besides the producer's
            ptx::mbar_init(&full_bar[s], 1 + 32 * GW);
            ptx::mbar_init(&empty_bar[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            ptx::mbar_init(&accf_bar[a], 1);
            // PAIR: the leader's MMA waits for the epilogues of both CTAs
            ptx::mbar_init(&acce_bar[a], PAIR ? 2 * C::kEpiWarps : C::kEpiWarps);
        }
        ptx::mbar_init(final_bar, 1);
        ptx::mbar_init(&metaf_bar[0], C::kEpiWarps);
        ptx::mbar_init(&metaf_bar[1], C::kEpiWarps);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    if (warp == 0 && lane < 2 + 2 * kNumBoxSizes) {
        const CUtensorMap* m = lane == 0   ? &args.tmA0
                               : lane == 1 ? &args.tmA1
                               : lane < 2 + kNumBoxSizes ? &args.tmB0[lane - 2]
                                                         : &args.tmB1[lane - 2 - kNumBoxSizes];
        ptx::prefetch_tmap(m);
    }
    if (warp == 1) {
        ptx::tmem_alloc<CG>(tmem_slot, C::kTmemCols);
        ptx::tmem_relinquish<CG>();
    }
    ptx::tc_fence_before();
    // PAIR: both CTAs' barriers and TMEM exist before either touches the other's
    if constexpr (PAIR) ptx::cluster_sync();
    else __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    // a tile covers 128 weight rows per sub-tile; gate/up sub-tiles are the two
    // matrices at the same rows, other sub-tiles are adjacent row blocks
    constexpr int kRowsPerTile = C::kSwiGLU ? 128 : 128 * MB;
    const int nblk_cta = (args.M_total + kRowsPerTile - 1) / kRowsPerTile;
    // PAIR: a tile is a pair of adjacent weight blocks, CTA r taking block 2p + r
    const int nblk = PAIR ? (nblk_cta + 1) / 2 : nblk_cta;
    // EPI_LOGITS may split K: tile t covers K part t % ksplit of tile t / ksplit
    const int ksplit = (EPI == EPI_LOGITS && args.k_splits > 1) ? args.k_splits : 1;
    const int total_tiles = ss.prefix[nseg] * nblk * ksplit;
    const int ksteps = args.K / C::kKStep;

    // K rotation of a tile (PAIR: of the pair's shared tile, so that both CTAs
    // fill every stage with the same K step)
    auto k_rot = [&](const TileInfo& ti, int span) -> int {
        if (!args.k_rotate) return 0;
        if constexpr (PAIR) {
            TileInfo tp = ti;
            tp.blk = ti.blk >> 1;
            return k_rotation(tp, span, nblk);
        } else {
            return k_rotation(ti, span, nblk_cta);
        }
    };
    auto fail = [&](int code) {
        *abort_flag = 1;
        set_device_error(args.status, code);
    };
    // tile t -> this CTA's share of it (all roles decode the same way)
    auto decode = [&](int t, TileInfo& ti) -> bool {
        if (!decode_tile(t / ksplit, nblk, nseg, ss, args.special_seg, ti)) return false;
        if constexpr (PAIR) {
            ti.blk = 2 * ti.blk + static_cast<int>(rank);
            ti.n_mma = (ti.n_valid + 31) & ~31;  // N split in two multiples of 16
        }
        return true;
    };

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        // Lane 0 waits for free slots and issues the bulk tensor copies.  For
        // a gathered tile (EPI_SWIGLU, ordinary segment, gather_tok set) the
        // whole warp also copies the token rows from the unpermuted source
        // with 16-byte cp.async: eight lanes per 128-byte row, written in the
        // same 128-byte-swizzled layout a tensor copy produces.
        const uint64_t pol_w =
            args.l2_hints ? ptx::policy_evict_first() : ptx::policy_evict_normal();
        const uint64_t pol_x =
            args.l2_hints ? ptx::policy_evict_last() : ptx::policy_evict_normal();
        // the special (shared-expert) segment's weights are re-read by every
        // token chunk of that segment: keep them in L2 rather than streaming
        const uint64_t pol_ws = pol_x;
        // weights of a routed segment with several token chunks
        const uint64_t pol_wm = !args.l2_hints                  ? ptx::policy_evict_normal()
                                : args.multi_chunk_policy == 2 ? ptx::policy_evict_last()
                                : args.multi_chunk_policy == 1 ? ptx::policy_evict_normal()
                                                               : pol_w;
        auto weight_policy = [&](const TileInfo& ti) -> uint64_t {
            if (ti.special) return pol_ws;
            return ss.prefix[ti.seg + 1] - ss.prefix[ti.seg] > 1 ? pol_wm : pol_w;
        };
        const bf16_raw_ptr gsrc = reinterpret_cast<bf16_raw_ptr>(args.gather_src);
        // token rows (and, for a gathered tile, their indices) come from
        // earlier launches
        ptx::grid_dep_wait();
        if (args.pdl_trigger_early) ptx::grid_dep_launch();
        uint32_t stage = 0, phase = 0;
        uint32_t armed = 0, armed_phase = 0;  // per-stage bits (lane 0)
        bool ok = true;
        for (int t = unit; ok && t < total_tiles; t += units) {
            TileInfo ti;
            const int ks = t % ksplit;
            if (!decode(t, ti)) continue;
            const int kb_begin = ks * ksteps / ksplit, kb_end = (ks + 1) * ksteps / ksplit;
            const int span = kb_end - kb_begin;
            const int rot = k_rot(ti, span);
            const CUtensorMap* tA = ti.special ? &args.tmA1 : &args.tmA0;
            const CUtensorMap* tB = ti.special ? args.tmB1 : args.tmB0;
            const int a_base = ti.special ? 0 : ti.seg * args.a_seg_stride;
            const uint64_t pw = weight_policy(ti);
            // (gathered rows: by the gather warps when GW > 0, bf16 or E4M3;
            // by this warp itself, bf16 only)
            const bool gather = C::kSwiGLU && (ET == 0 || GW > 0) && !PAIR &&
                                args.gather_tok != nullptr && !ti.special;
            // GW > 0: the gather warps copy the rows; this warp only the weights
            const bool own_gather = gather && GW == 0;
            // token rows this CTA loads (PAIR: its half of the tile's columns)
            const int b_rows = PAIR ? ti.n_mma / 2 : ti.n_mma;
            const int b_row0 = ti.b_row + (PAIR ? static_cast<int>(rank) * b_rows : 0);
            if (own_gather) {
                __syncwarp();  // the previous tile's rows are all issued
                for (int i = lane; i < ti.n_mma; i += 32) {
                    const int tok = i < ti.n_valid ? __ldg(args.gather_tok + ti.b_row + i) : -1;
                    // padding rows (never stored) and out-of-range indices: a row of zeros
                    s_goff[i] = static_cast<unsigned>(tok) < static_cast<unsigned>(args.n_tokens)
                                    ? static_cast<int64_t>(tok) * args.K
                                    : int64_t(-1);
                }
                __syncwarp();
            }
            // expected bytes (PAIR: the leader expects both CTAs' copies)
            const uint32_t bytes =
                PAIR ? 2u * (C::kABytes + b_rows * 128) : C::kABytes + (gather ? 0 : ti.n_mma * 128);
            // (gathered rows arrive through cp.async, counted as arrivals)
            for (int i = 0; i < span; ++i) {
                const int kb = kb_begin + (i + rot < span ? i + rot : i + rot - span);
                int got = 1;
                if (lane == 0) got = ptx::mbar_wait(&empty_bar[stage], phase ^ 1, abort_flag);
                got = __shfl_sync(0xffffffffu, got, 0);
                if (!got) {
                    if (lane == 0) fail(DEV_ERR_TIMEOUT);
                    ok = false;
                    break;
                }
                uint8_t* sA = ring + stage * C::kStageBytes;
                uint8_t* sB = sA + C::kABytes;
                const int k0 = kb * C::kKStep;
                if (own_gather) {
                    // lane: 16-byte chunk (lane & 7) of rows lane/8 + 4i; the
                    // offsets of four rows are read before their copies are
                    // issued (each copy is ordered against later loads)
                    const int chunk = lane & 7;
                    const bf16_raw_ptr base = gsrc + k0 + chunk * 8;
                    for (int r0 = 0; r0 < ti.n_mma; r0 += 16) {  // n_mma: a multiple of 16
                        int64_t off[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j) off[j] = s_goff[r0 + (lane >> 3) + 4 * j];
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const int r = r0 + (lane >> 3) + 4 * j;
                            ptx::cp_async_16(sB + r * 128 + ((chunk ^ (r & 7)) << 4),
                                             off[j] >= 0 ? static_cast<const void*>(base + off[j])
                                                         : static_cast<const void*>(gsrc),
                                             off[j] >= 0 ? 16u : 0u);
                        }
                    }
                    ptx::cp_async_mbar_arrive(&full_bar[stage]);
                    __syncwarp();  // every lane's arrival is counted before lane 0 arrives
                }
                if (lane == 0) {
                    // completion is counted on this CTA's barrier, or (PAIR) on
                    // the leader's, which alone expects the bytes
                    uint32_t bar = ptx::smem_u32(&full_bar[stage]);
                    if constexpr (PAIR) bar = ptx::mapa_shared(bar, 0);
                    if (!PAIR || rank == 0) {
                        ptx::mbar_arrive_expect_tx(&full_bar[stage], bytes);
                        armed |= 1u << stage;
                        armed_phase = (armed_phase & ~(1u << stage)) | (phase << stage);
                    }
                    auto load2d = [&](void* dst, const CUtensorMap* m, int c0, int c1,
                                      uint64_t pol) {
                        if constexpr (PAIR) ptx::tma_load_2d_pair(dst, m, c0, c1, bar, pol);
                        else ptx::tma_load_2d(dst, m, c0, c1, &full_bar[stage], pol);
                    };
                    auto load3d = [&](void* dst, const CUtensorMap* m, int c0, int c1, int c2,
                                      uint64_t pol) {
                        if constexpr (PAIR) ptx::tma_load_3d_pair(dst, m, c0, c1, c2, bar, pol);
                        else ptx::tma_load_3d(dst, m, c0, c1, c2, &full_bar[stage], pol);
                    };
                    if constexpr (C::kDown) {
                        // MN-major A: one 3D copy of the tile's 128-byte-wide H
                        // chunks (bf16: 2*MB chunks of 64 values x 64 K-rows;
                        // FP8: MB chunks of 128 values x 128 K-rows; TF32:
                        // 4*MB chunks of 32 values x 32 K-rows), chunk-major
                        load3d(sA, tA, 0, a_base + args.a_off0 + k0, ti.blk * (C::kElemBytes * MB),
                               pw);
                    } else if constexpr (C::kSwiGLU) {
                        // gate and up tiles (adjacent matrices) in one 3D copy
                        load3d(sA, tA, k0, ti.blk * 128, a_base + args.a_off0, pw);
                    } else if constexpr (MB == 2) {
                        // both 128-row blocks in one 256-row box
                        load2d(sA, tA, k0, a_base + args.a_off0 + ti.blk * 256, pw);
                    } else {
                        load2d(sA, tA, k0, a_base + args.a_off0 + ti.blk * 128, pw);
                    }
                    if (!gather) {
                        int q = 0;
#pragma unroll
                        for (int j = kNumBoxSizes - 1; j >= 0; --j) {
                            if ((b_rows >> 4) & (1 << j)) {
                                load2d(sB + q * 128, &tB[j], k0, b_row0 + q, pol_x);
                                q += 16 << j;
                            }
                        }
                    }
                }
                if (++stage == C::kStages) {
                    stage = 0;
                    phase ^= 1;
                }
            }
        }
        // every copy of this CTA is issued: the next launch may start
        if (!args.pdl_trigger_early) ptx::grid_dep_launch();
        // never leave with copies still writing into this CTA's shared memory
        ptx::cp_async_wait_all();
        __syncwarp();
        if (lane == 0) {
            for (int s = 0; s < C::kStages; ++s) {
                if (armed & (1u << s)) {
                    ptx::mbar_wait(&full_bar[s], (armed_phase >> s) & 1u, nullptr);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // (PAIR: the leader only; its cta_group::2 MMAs span both CTAs)
        if (lane == 0 && rank == 0) {
            uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
            bool ok = true;
            constexpr uint32_t kAMajor = C::kDown ? 1u : 0u;
            // MN-major A: per MMA (32 bytes of K: 16 bf16 / 32 FP8 / 8 TF32)
            // the next 16 / 32 / 8 K-rows of 128 bytes; between 128-byte H
            // chunks one stage's K-rows: 8 KB (bf16: two chunks per 128-row
            // sub-tile), 4 KB (TF32: four chunks) -- unused for FP8, where one
            // chunk is the 128 rows.  TF32 tiles use the 128-byte swizzle with
            // 32-byte atoms (the copies write it; see make_tmap_down)
            constexpr uint32_t kMnStep = 4096u / C::kElemBytes;
            constexpr uint32_t kMnLbo = 16384u / C::kElemBytes;
            // PAIR: arrive on the barrier at the same offset in both CTAs
            auto commit = [&](uint64_t* bar) {
                if constexpr (PAIR) {
                    const uint32_t own = ptx::smem_u32(bar);
                    ptx::mma_commit_pair(own);
                    ptx::mma_commit_pair(ptx::mapa_shared(own, 1));
                } else {
                    ptx::mma_commit(bar);
                }
            };
            constexpr uint32_t kM = PAIR ? 256u : 128u;
            for (int t = unit; ok && t < total_tiles; t += units) {
                TileInfo ti;
                const int ks = t % ksplit;
                if (!decode(t, ti)) continue;
                const int span = (ks + 1) * ksteps / ksplit - ks * ksteps / ksplit;
                if (!ptx::mbar_wait(&acce_bar[acc], acc_phase ^ 1, abort_flag)) {
                    fail(DEV_ERR_TIMEOUT);
                    break;
                }
                ptx::tc_fence_after();
                const uint32_t d0 = tmem_base + acc * C::kAccCols;
                const uint32_t idesc = FP8    ? ptx::idesc_e4m3_f32(kM, ti.n_mma, kAMajor, 0)
                                       : TF32 ? ptx::idesc_tf32_f32(kM, ti.n_mma, kAMajor, 0)
                                              : ptx::idesc_bf16_f32(kM, ti.n_mma, kAMajor, 0);
                for (int i = 0; i < span; ++i) {
                    if (!ptx::mbar_wait(&full_bar[stage], phase, abort_flag)) {
                        fail(DEV_ERR_TIMEOUT);
                        ok = false;
                        break;
                    }
                    // token rows gathered with cp.async were written through
                    // the generic proxy; the MMA reads them through the async one
                    if constexpr (C::kSwiGLU) ptx::fence_proxy_async_smem();
                    ptx::tc_fence_after();
                    const uint32_t a_addr = ptx::smem_u32(ring + stage * C::kStageBytes);
                    const uint32_t b_addr = a_addr + C::kABytes;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint32_t accum = (i > 0 || kk > 0) ? 1u : 0u;
                        const uint64_t bdesc = ptx::smem_desc_sw128(b_addr + kk * 32, 16, 1024);
#pragma unroll
                        for (int j = 0; j < MB; ++j) {
                            const uint32_t a_sub = a_addr + j * C::kATileBytes;
                            // (TF32 MN-major: the 32-byte-atom swizzle, 4-row K groups)
                            const uint64_t adesc =
                                !C::kDown ? ptx::smem_desc_sw128(a_sub + kk * 32, 16, 1024)
                                : TF32    ? ptx::smem_desc_sw128_32b(a_sub + kk * kMnStep, kMnLbo, 512)
                                          : ptx::smem_desc_sw128(a_sub + kk * kMnStep, kMnLbo, 1024);
                            if constexpr (FP8)
                                ptx::mma_fp8<CG>(d0 + j * NMAX, adesc, bdesc, idesc, accum);
                            else if constexpr (TF32)
                                ptx::mma_tf32<CG>(d0 + j * NMAX, adesc, bdesc, idesc, accum);
                            else
                                ptx::mma_bf16<CG>(d0 + j * NMAX, adesc, bdesc, idesc, accum);
                        }
                    }
                    commit(&empty_bar[stage]);
                    if (++stage == C::kStages) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (!ok) break;
                commit(&accf_bar[acc]);
                if (++acc == C::kAccStages) {
                    acc = 0;
                    acc_phase ^= 1;
                }
            }
            // all issued MMAs must retire before TMEM is released
            if constexpr (PAIR) ptx::mma_commit_pair(ptx::smem_u32(final_bar));
            else ptx::mma_commit(final_bar);
            ptx::mbar_wait(final_bar, 0, nullptr);
        }
    } else if (GW > 0 && warp >= 2 + C::kEpiWarps) {
        // ------------------------------------------------------------ row gather
        // gather warp gw copies the 16-row groups gw, gw + GW, ... of each
        // gathered tile (lane: 16-byte chunk lane & 7 of rows lane/8 + 4j of a
        // group) and arrives once per stage on the full barrier, when its
        // copies have landed (at once for tiles it has no rows of)
        const int gw = warp - 2 - C::kEpiWarps;
        // (byte addressing: a stage holds 128 bytes of every row, 64 bf16 or
        // 128 E4M3 values)
        const uint8_t* gsrc = static_cast<const uint8_t*>(args.gather_src);
        ptx::grid_dep_wait();  // the row indices come from an earlier launch
        uint32_t stage = 0, phase = 0;
        bool ok = true;
        for (int t = unit; ok && t < total_tiles; t += units) {
            TileInfo ti;
            const int ks = t % ksplit;
            if (!decode(t, ti)) continue;
            const int kb_begin = ks * ksteps / ksplit, kb_end = (ks + 1) * ksteps / ksplit;
            const int span = kb_end - kb_begin;
            const int rot = k_rot(ti, span);
            const bool gather = args.gather_tok != nullptr && !ti.special;
            const int ngroups = ti.n_mma >> 4;
            if (gather) {
                __syncwarp();  // this warp's previous rows are all issued
                for (int g = gw; g < ngroups; g += GW) {
                    for (int i = lane; i < 16; i += 32) {
                        const int r = g * 16 + i;
                        const int tok =
                            r < ti.n_valid ? __ldg(args.gather_tok + ti.b_row + r) : -1;
                        s_goff[r] = static_cast<unsigned>(tok) <
                                            static_cast<unsigned>(args.n_tokens)
                                        ? static_cast<int64_t>(tok) * args.K * C::kElemBytes
                                        : int64_t(-1);
                    }
                }
                __syncwarp();
            }
            for (int i = 0; i < span; ++i) {
                const int kb = kb_begin + (i + rot < span ? i + rot : i + rot - span);
                int got = 1;
                if (lane == 0) got = ptx::mbar_wait(&empty_bar[stage], phase ^ 1, abort_flag);
                got = __shfl_sync(0xffffffffu, got, 0);
                if (!got) {
                    ok = false;
                    break;
                }
                if (gather) {
                    uint8_t* sB = ring + stage * C::kStageBytes + C::kABytes;
                    const int chunk = lane & 7;
                    const uint8_t* base = gsrc + kb * 128 + chunk * 16;
                    for (int g = gw; g < ngroups; g += GW) {
                        const int r0 = g * 16;
                        int64_t off[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j) off[j] = s_goff[r0 + (lane >> 3) + 4 * j];
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const int r = r0 + (lane >> 3) + 4 * j;
                            ptx::cp_async_16(sB + r * 128 + ((chunk ^ (r & 7)) << 4),
                                             off[j] >= 0 ? static_cast<const void*>(base + off[j])
                                                         : static_cast<const void*>(gsrc),
                                             off[j] >= 0 ? 16u : 0u);
                        }
                    }
                }
                ptx::cp_async_mbar_arrive_noinc(&full_bar[stage]);
                if (++stage == C::kStages) {
                    stage = 0;
                    phase ^= 1;
                }
            }
        }
        ptx::cp_async_wait_all();  // nothing still writing into shared memory
    } else {
        // ------------------------------------------------------------ epilogue
        const int quarter = warp & 3;
        const int half = (warp - 2) >> 2;  // which of the two warps on this quarter
        const int row_in_tile = quarter * 32 + lane;
        ptx::grid_dep_wait();  // row metadata and outputs are shared with earlier launches
        uint32_t acc = 0, acc_phase = 0;
        uint32_t mi = 0, meta_phase = 0;
        // hands accumulator buffer `acc` back to the MMA warp once this warp's
        // TMEM reads of it have completed (PAIR: on the leader CTA, which
        // waits for both CTAs)
        auto release_acc = [&]() {
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if constexpr (PAIR)
                    ptx::mbar_arrive_cluster(ptx::mapa_shared(ptx::smem_u32(&acce_bar[acc]), 0));
                else
                    ptx::mbar_arrive(&acce_bar[acc]);
            }
        };
        for (int t = unit; t < total_tiles; t += units) {
            TileInfo ti;
            const int ks = t % ksplit;
            if (!decode(t, ti)) continue;
            int32_t* w_tok = reinterpret_cast<int32_t*>(s_meta) + mi * 2 * NMAX;
            float* w_wt = reinterpret_cast<float*>(w_tok + NMAX);
            if constexpr (C::kMeta) {
                // token and routing weight of every column, fetched by the
                // epilogue warps together before the accumulator is ready, so
                // the loads overlap the main loop.  Two buffers alternate by
                // tile; a warp only refills a buffer after all epilogue warps
                // have published their part of the next tile, i.e. after all
                // of them finished reading it.
                for (int c = (warp - 2) * 32 + lane; c < ti.n_valid; c += 32 * C::kEpiWarps) {
                    const int r = ti.out_row + c;
                    int tok;
                    float wt;
                    if (r < args.routed_rows) {
                        tok = args.row_token ? __ldg(args.row_token + r) : r;
                        wt = args.row_weight ? __ldg(args.row_weight + r) : 1.0f;
                    } else {
                        tok = r - args.routed_rows;
                        wt = 1.0f;
                    }
                    if (args.token_scale) wt *= __ldg(args.token_scale + tok);
                    w_tok[c] = tok;
                    w_wt[c] = wt;
                }
                __syncwarp();
                if (lane == 0) ptx::mbar_arrive(&metaf_bar[mi]);
                if (!ptx::mbar_wait(&metaf_bar[mi], meta_phase, abort_flag)) {
                    fail(DEV_ERR_TIMEOUT);
                    break;
                }
                mi ^= 1;
                if (mi == 0) meta_phase ^= 1;
            }
            // FP8 channel scales of this lane's rows, fetched before the
            // accumulator is ready (under the main loop): gate/up: the gate
            // and up scales of row m; down: h scale x weight-column scale of
            // each sub-tile's row
            static_assert(MB <= 2, "at most two 128-row sub-tiles");
            float ch0 = 1.0f, ch1 = 1.0f;
            if constexpr (FP8 && C::kSwiGLU) {
                const int m = ti.blk * 128 + row_in_tile;
                const float* sc = ti.special ? args.scale_w_special
                                             : args.scale_w + static_cast<size_t>(ti.seg) * 2 *
                                                                  args.M_total;
                if (m < args.M_total) {
                    ch0 = __ldg(sc + m);
                    ch1 = __ldg(sc + args.M_total + m);
                }
            } else if constexpr (FP8 && C::kDown) {
                const float* sc = ti.special ? args.scale_w_special
                                             : args.scale_w + static_cast<size_t>(ti.seg) *
                                                                  args.M_total;
                const int m0 = ti.blk * MB * 128 + row_in_tile;
                if (m0 < args.M_total) ch0 = args.h_scale * __ldg(sc + m0);
                if (MB > 1 && m0 + 128 < args.M_total) ch1 = args.h_scale * __ldg(sc + m0 + 128);
            }
            if (!ptx::mbar_wait(&accf_bar[acc], acc_phase, abort_flag)) {
                fail(DEV_ERR_TIMEOUT);
                break;
            }
            ptx::tc_fence_after();
            const uint32_t tbase = tmem_base + acc * C::kAccCols +
                                   (static_cast<uint32_t>(quarter * 32) << 16);
            if constexpr (C::kSwiGLU) {
                // h = silu(clamp(g)) * clamp(u) on this warp's 16-column chunks;
                // the next chunk's TMEM loads are in flight while one is
                // computed.
                const int m = ti.blk * 128 + row_in_tile;
                const bool m_ok = m < args.M_total;
                __nv_bfloat16* hout = reinterpret_cast<__nv_bfloat16*>(args.out);
                const float sg = ch0, su = ch1;  // FP8: gate and up channel scales
                auto emit = [&](float (&g)[16], float (&u)[16], int c0) {
                    float hv[16];
                    float ts16[16];  // FP8 token scales, read before the stores
                    if constexpr (FP8) {
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const float4 t4 = reinterpret_cast<const float4*>(w_wt + c0)[q];
                            ts16[4 * q] = t4.x;
                            ts16[4 * q + 1] = t4.y;
                            ts16[4 * q + 2] = t4.z;
                            ts16[4 * q + 3] = t4.w;
                        }
                    }
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        float gin = g[j], uin = u[j];
                        if constexpr (FP8) {
                            // token scale (per column) x channel scale (per lane)
                            const float ts = ts16[j];
                            gin *= ts * sg;
                            uin *= ts * su;
                        }
                        const float gg = clamp_keep_nan(gin, args.clip);
                        const float uu = clamp_keep_nan(uin, args.clip);
                        // silu(g) = g / (1 + e^-g): approximate exp2 and
                        // reciprocal (both ~1e-7 relative, far below bf16)
                        hv[j] = gg * fast_rcp(1.0f + __expf(-gg)) * uu;
                        if constexpr (FP8) hv[j] *= args.h_scale_inv;  // exact: power of two
                    }
                    if constexpr (TF32) {
                        // fp32 h: each lane stores its own row's value; the 32
                        // lanes of a column write 128 consecutive bytes
                        float* hf = reinterpret_cast<float*>(args.out);
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            if (m_ok && c0 + j < ti.n_valid)
                                hf[static_cast<size_t>(ti.out_row + c0 + j) * args.out_ld + m] =
                                    hv[j];
                        }
                        return;
                    }
                    // lane pairs (I is a multiple of 64: a pair agrees on m_ok)
                    const bool odd = lane & 1;
                    const size_t ld = static_cast<size_t>(args.out_ld);
                    const size_t row0 = static_cast<size_t>(ti.out_row + c0) * ld + (m & ~1);
                    auto ok = [&](int r) { return m_ok && c0 + r < ti.n_valid; };
                    if constexpr (FP8)
                        store_pairs_e4m3(reinterpret_cast<uint8_t*>(args.out), row0, ld, hv, odd, ok);
                    else
                        store_pairs_bf16(hout, row0, ld, hv, odd, ok);
                };
                float g0[16], u0[16], g1[16], u1[16];
                int c0 = half * 16;  // this warp's chunks: c0, c0 + 32, ...
                if (c0 < ti.n_mma) {
                    ptx::tmem_ld16(tbase + c0, g0);
                    ptx::tmem_ld16(tbase + NMAX + c0, u0);
                    ptx::tmem_ld_wait();
                    ptx::reg_fence(g0);
                    ptx::reg_fence(u0);
                }
                for (; c0 < ti.n_mma; c0 += 64) {
                    const bool more1 = c0 + 32 < ti.n_mma;
                    if (more1) {
                        ptx::tmem_ld16(tbase + c0 + 32, g1);
                        ptx::tmem_ld16(tbase + NMAX + c0 + 32, u1);
                    }
                    emit(g0, u0, c0);
                    if (!more1) break;
                    ptx::tmem_ld_wait();
                    ptx::reg_fence(g1);
                    ptx::reg_fence(u1);
                    const bool more2 = c0 + 64 < ti.n_mma;
                    if (more2) {
                        ptx::tmem_ld16(tbase + c0 + 64, g0);
                        ptx::tmem_ld16(tbase + NMAX + c0 + 64, u0);
                    }
                    emit(g1, u1, c0 + 32);
                    if (!more2) break;
                    ptx::tmem_ld_wait();
                    ptx::reg_fence(g0);
                    ptx::reg_fence(u0);
                }
            } else {
                // Per sub-tile, this warp's 16-column chunks are read from TMEM
                // in batches of up to five (80 registers) behind one wait.  The
                // down GEMMs hand the accumulator back to the MMA warp as soon
                // as their last batch is in registers, so the next tile's MMAs
                // run under the scaling and stores of that batch.
                constexpr int kCW = (NMAX + 31) / 32;       // chunks per warp and sub-tile
                constexpr int kNB = (kCW + 4) / 5;          // batches per sub-tile
                constexpr int kBC = (kCW + kNB - 1) / kNB;  // chunks per batch
                auto emit_chunk = [&](const float (&v)[16], int c0, int m, bool m_ok,
                                      float lane_scale) {
                    // The chunk's column weights (and tokens) are read into
                    // registers before its first store: the output pointer is
                    // generic, so a read of the metadata placed after a store
                    // could not be moved above it and every column would wait
                    // out a full memory round trip.
                    float cw[16];
                    if constexpr (C::kMeta) {
                        // (16-byte loads: the metadata buffers and c0 are
                        // 64-byte aligned)
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            const float4 w4 = reinterpret_cast<const float4*>(w_wt + c0)[q];
                            cw[4 * q] = w4.x;
                            cw[4 * q + 1] = w4.y;
                            cw[4 * q + 2] = w4.z;
                            cw[4 * q + 3] = w4.w;
                        }
                    }
                    if constexpr (EPI == EPI_DOWN_ATOMIC) {
                        float* oacc = reinterpret_cast<float*>(args.out);
                        // each accumulator element takes top_k + 1 additions spread
                        // over the whole launch: keep its lines in L2 between them
                        const uint64_t pol_acc = args.l2_hints ? ptx::policy_evict_last()
                                                               : ptx::policy_evict_normal();
                        int ct[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) ct[j] = w_tok[c0 + j];
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const int c = c0 + j;
                            if (m_ok && c < ti.n_valid) {
                                const int tok = ct[j];
                                if (static_cast<unsigned>(tok) <
                                    static_cast<unsigned>(args.n_tokens)) {
                                    ptx::red_add_f32(
                                        oacc + static_cast<size_t>(tok) * args.out_ld + m,
                                        cw[j] * v[j], pol_acc);
                                } else {
                                    set_device_error(args.status, DEV_ERR_BAD_INDEX);
                                }
                            }
                        }
                    } else if (EPI == EPI_DOWN_STORE && !args.out_f32) {
                        // weighted bf16 rows, stored by lane pairs (H is a
                        // multiple of 64: a pair agrees on m_ok)
                        float a[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) a[j] = v[j] * lane_scale * cw[j];
                        const size_t ld = static_cast<size_t>(args.out_ld);
                        const size_t row0 =
                            static_cast<size_t>(ti.out_row + c0) * ld + (m & ~1);
                        store_pairs_bf16(reinterpret_cast<__nv_bfloat16*>(args.out), row0, ld, a,
                                         (lane & 1) != 0,
                                         [&](int r) { return m_ok && c0 + r < ti.n_valid; });
                    } else if (m_ok) {
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            if (c0 + j < ti.n_valid) {
                                const size_t o =
                                    static_cast<size_t>(ti.out_row + c0 + j) * args.out_ld + m;
                                if constexpr (EPI == EPI_LOGITS) {
                                    reinterpret_cast<float*>(args.out)[o + ks * args.split_stride] =
                                        v[j];
                                } else {
                                    reinterpret_cast<float*>(args.out)[o] = v[j] * cw[j];
                                }
                            }
                        }
                    }
                };
#pragma unroll 1
                for (int sub = 0; sub < MB; ++sub) {
                    const int m = (ti.blk * MB + sub) * 128 + row_in_tile;
                    const bool m_ok = m < args.M_total;
                    // FP8: h scale x this lane's weight-column scale
                    const float lane_scale = sub == 0 ? ch0 : ch1;
#pragma unroll 1
                    for (int b = 0; b < kNB; ++b) {
                        float v[kBC][16];
#pragma unroll
                        for (int i = 0; i < kBC; ++i) {
                            const int c0 = half * 16 + 32 * (b * kBC + i);
                            if (c0 < ti.n_mma) ptx::tmem_ld16(tbase + sub * NMAX + c0, v[i]);
                        }
                        ptx::tmem_ld_wait();
#pragma unroll
                        for (int i = 0; i < kBC; ++i) ptx::reg_fence(v[i]);
                        if (C::kDown && sub == MB - 1 && b == kNB - 1) release_acc();
#pragma unroll
                        for (int i = 0; i < kBC; ++i) {
                            const int c0 = half * 16 + 32 * (b * kBC + i);
                            if (c0 < ti.n_mma) emit_chunk(v[i], c0, m, m_ok, lane_scale);
                        }
                    }
                }
            }
            if constexpr (!C::kDown) release_acc();
            if (++acc == C::kAccStages) {
                acc = 0;
                acc_phase ^= 1;
            }
        }
    }

    ptx::tc_fence_before();
    // PAIR: neither CTA leaves (or frees TMEM) while the other may still signal
    // its barriers or the leader's MMAs may still write its TMEM
    if constexpr (PAIR) ptx::cluster_sync();
    else __syncthreads();
    ptx::tc_fence_after();
    if (warp == 1) ptx::tmem_dealloc<CG>(tmem_base, C::kTmemCols);

    if constexpr (EPI == EPI_LOGITS) {
        if (args.route_idx != nullptr) {
            // fused routing: this CTA ran exactly tile blockIdx.x (nblk == 1)
            const int ks = static_cast<int>(blockIdx.x) % ksplit;
            const int chunk = static_cast<int>(blockIdx.x) / ksplit;
            __threadfence();  // this CTA's partial logits, before the count below
            __syncthreads();
            if (threadIdx.x == 0) {
                atomicAdd(args.route_count + chunk, 1);
                const int go = ptx::wait_counter_at_least(args.route_count + chunk, ksplit) ? 1 : 0;
                if (!go) set_device_error(args.status, DEV_ERR_TIMEOUT);
                *route_go = go;
            }
            __syncthreads();
            if (*route_go) {
                const int cl = args.single_chunk_len;
                const int64_t r0 = static_cast<int64_t>(chunk) * cl;
                const int64_t rows = min(static_cast<int64_t>(cl), args.single_rows - r0);
                const int64_t share = (rows + ksplit - 1) / ksplit;
                const int64_t a = r0 + ks * share;
                const int64_t b = min(r0 + rows, a + share);
                for (int64_t t = a + warp; t < b; t += blockDim.x >> 5)
                    route_one_token(reinterpret_cast<float*>(args.out), ksplit, args.split_stride,
                                    args.route_keep_sum != 0, args.route_bias, t, args.M_total,
                                    args.route_k, args.route_scale, args.route_idx, args.route_w);
            }
        }
    }
}

}  // namespace moe
