// moe_api.cu -- host side of the C ABI declared in include/moe.h:
// argument validation, workspace carving, TMA tensor-map encoding, kernel
// launch sequencing, the launch counter and the per-kernel event profiler.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <utility>
#include <vector>

#include "../../include/moe.h"
#include "gemm_sm100.cuh"
#include "small_kernels.cuh"

namespace moe {
namespace {

// ------------------------------------------------------------------ launch bookkeeping

std::atomic<int64_t> g_launches{0};

struct ProfRecord {
    const char* name;
    cudaEvent_t start, stop;
};

struct Profiler {
    std::mutex mu;
    bool on = false;
    std::vector<cudaEvent_t> pool;  // 2 per record
    std::vector<ProfRecord> recs;
    size_t cap = 0;
};
Profiler g_prof;

struct LaunchScope {
    cudaEvent_t stop = nullptr;
    cudaStream_t stream;
    LaunchScope(const char* name, cudaStream_t s) : stream(s) {
        if (!g_prof.on) return;
        std::lock_guard<std::mutex> lk(g_prof.mu);
        if (!g_prof.on || g_prof.recs.size() >= g_prof.cap) return;
        ProfRecord r{name, g_prof.pool[2 * g_prof.recs.size()],
                     g_prof.pool[2 * g_prof.recs.size() + 1]};
        cudaEventRecord(r.start, s);
        stop = r.stop;
        g_prof.recs.push_back(r);
    }
    ~LaunchScope() {
        g_launches.fetch_add(1, std::memory_order_relaxed);
        if (stop) cudaEventRecord(stop, stream);
    }
};

#define MOE_LAUNCH(name, stream, ...)              \
    do {                                           \
        LaunchScope scope_(name, stream);          \
        __VA_ARGS__;                               \
        cudaError_t e_ = cudaGetLastError();       \
        if (e_ != cudaSuccess) return MOE_ERR_CUDA; \
    } while (0)

// ------------------------------------------------------------------ device info

int sm_count() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    static int cache[64] = {0};
    if (dev < 64 && cache[dev]) return cache[dev];
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
    if (dev < 64) cache[dev] = n;
    return n;
}

// ------------------------------------------------------------------ tensor maps

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess) {
            fn = reinterpret_cast<EncodeTiledFn>(p);
        }
    });
    return fn;
}

// Element type of a tensor map: bf16 (2 bytes) or FP8 codes (1 byte).  A
// 128-byte swizzled row holds 128 / bytes elements.
struct ElemType {
    CUtensorMapDataType dt;
    int bytes;
};
constexpr ElemType kBF16{CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2};
constexpr ElemType kU8{CU_TENSOR_MAP_DATA_TYPE_UINT8, 1};
constexpr ElemType kF32{CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4};

int env_int(const char* name, int dflt);

// L2 sector promotion of the expert-weight tensor maps (MOE_L2_PROMO: 0 none,
// 1 64 B, 2 128 B, 3 256 B; default 256 B).  A weight tile row is 128 bytes
// per pipeline stage; with 256-byte promotion the next stage's 128 bytes of
// the same row come in with it.
CUtensorMapL2promotion weight_l2_promotion() {
    const int v = env_int("MOE_L2_PROMO", 3);
    switch (v) {
        case 0: return CU_TENSOR_MAP_L2_PROMOTION_NONE;
        case 1: return CU_TENSOR_MAP_L2_PROMOTION_L2_64B;
        case 2: return CU_TENSOR_MAP_L2_PROMOTION_L2_128B;
        default: return CU_TENSOR_MAP_L2_PROMOTION_L2_256B;
    }
}

// 2D row-major [rows, cols] tensor, box = one 128-byte row segment x box_rows
// rows, 128-byte swizzle, zero fill outside the tensor.
bool make_tmap(CUtensorMap* m, const void* ptr, int64_t rows, int64_t cols, int box_rows,
               ElemType et = kBF16) {
    EncodeTiledFn fn = encode_fn();
    if (!fn || rows <= 0 || cols <= 0) return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * et.bytes};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / et.bytes),
                         static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = fn(m, et.dt, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Gate/up weights as a 3D bf16 tensor {H, I, n_mats} (n_mats [I,H] matrices
// back to back), box {64, 128, 2}: one copy brings the gate and the up tile.
bool make_tmap_gateup(CUtensorMap* m, const void* ptr, int64_t n_mats, int64_t I, int64_t H,
                      ElemType et = kBF16) {
    EncodeTiledFn fn = encode_fn();
    if (!fn || n_mats <= 0) return false;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(I),
                          static_cast<cuuint64_t>(n_mats)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(H) * et.bytes,
                             static_cast<cuuint64_t>(I * H) * et.bytes};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / et.bytes), 128u, 2u};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    CUresult r = fn(m, et.dt, 3, const_cast<void*>(ptr), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    weight_l2_promotion(), CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Down-projection weights [rows, H] (H contiguous) as a 3D tensor {c, rows,
// H/c} with c = 128 bytes of H values (64 bf16, 128 E4M3, 32 fp32): dim 0 = c
// consecutive H values, dim 1 = the row, dim 2 = which c-wide H chunk (stride
// 128 bytes).  A {c, c, bytes*mb} box is one K-step of the chunks of mb
// 128-row sub-tiles, laid out chunk by chunk in shared memory.
bool make_tmap_down(CUtensorMap* m, const void* ptr, int64_t rows, int64_t H, int mb,
                    ElemType et = kBF16) {
    EncodeTiledFn fn = encode_fn();
    const int64_t chunk = 128 / et.bytes;  // H values per 128-byte chunk
    if (!fn || rows <= 0 || H % chunk != 0) return false;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(chunk), static_cast<cuuint64_t>(rows),
                          static_cast<cuuint64_t>(H / chunk)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(H) * et.bytes, 128u};
    // one K-step: 64 (bf16) or 128 (FP8) rows of each of the tile's chunks
    cuuint32_t box[3] = {static_cast<cuuint32_t>(chunk), static_cast<cuuint32_t>(chunk),
                         static_cast<cuuint32_t>(et.bytes * mb)};
    cuuint32_t estr[3] = {1u, 1u, 1u};
    // fp32 (TF32) MN-major operands take the 128-byte swizzle with 32-byte
    // atoms, the only MN-major shared-memory layout TF32 MMAs accept
    const CUtensorMapSwizzle sw =
        et.bytes == 4 ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B : CU_TENSOR_MAP_SWIZZLE_128B;
    CUresult r = fn(m, et.dt, 3, const_cast<void*>(ptr), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                    weight_l2_promotion(), CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// The token-row operand with the five box heights 16 << j.
bool make_tmap_rows(CUtensorMap* maps, const void* ptr, int64_t rows, int64_t cols,
                    ElemType et = kBF16) {
    for (int j = 0; j < kNumBoxSizes; ++j)
        if (!make_tmap(&maps[j], ptr, rows, cols, 16 << j, et)) return false;
    return true;
}

// ------------------------------------------------------------------ problem checks

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int32_t check_problem(const moe_problem* p) {
    if (!p) return MOE_ERR_INVALID_ARG;
    if (p->T < 0) return MOE_ERR_INVALID_ARG;
    if (p->dtype != MOE_F32 && p->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
    if (p->H < 64 || p->H % 64 != 0 || p->I < 64 || p->I % 64 != 0) return MOE_ERR_UNSUPPORTED;
    // top_k <= 32: the router and the row gather keep one selection per lane
    if (p->E < 1 || p->E > kMaxExperts || p->top_k < 1 || p->top_k > p->E || p->top_k > 32)
        return MOE_ERR_UNSUPPORTED;
    if (p->num_shared != 0 && p->num_shared != 1) return MOE_ERR_UNSUPPORTED;
    if (p->T * static_cast<int64_t>(p->top_k + p->num_shared) >= (int64_t(1) << 31))
        return MOE_ERR_UNSUPPORTED;
    if (static_cast<int64_t>(p->E) * 3 * p->I >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED;
    if (!std::isfinite(p->routed_scale)) return MOE_ERR_INVALID_ARG;
    if (std::isnan(p->clip_limit)) return MOE_ERR_INVALID_ARG;
    return MOE_OK;
}

float effective_clip(const moe_problem* p) {
    return (p->clip_limit > 0.0f && std::isfinite(p->clip_limit)) ? p->clip_limit : INFINITY;
}


int env_int(const char* name, int dflt) {
    const char* e = std::getenv(name);
    return e ? std::atoi(e) : dflt;
}

bool nmax_supported(int n) {
    return n == 16 || n == 32 || n == 64 || n == 128 || n == 160 || n == 256;
}

// Token-row tile width (MMA N) of the expert GEMMs, from the mean rows per
// expert: small batches get narrow tiles (deep weight pipelines, little
// padding); prefill-sized experts (~100-200 rows) get 160, which leaves room
// for a 4-deep pipeline of gate+up weight tiles; larger segments get 256.
// MOE_NMAX in the environment overrides it (tuning knob).
int pick_nmax(double mean_rows) {
    const int forced = [] {
        const int v = env_int("MOE_NMAX", 0);
        return nmax_supported(v) ? v : 0;
    }();
    if (forced) return forced;
    if (mean_rows >= 200.0) return 256;
    if (mean_rows >= 96.0) return 160;
    if (mean_rows >= 48.0) return 128;
    if (mean_rows >= 24.0) return 64;
    if (mean_rows >= 12.0) return 32;
    return 16;
}

// Token-row tile width of the down GEMM: the gate/up width (narrower tiles
// re-read the weights more often, which costs power under the 1 kW cap more
// than the double-buffered accumulator gains).  MOE_DOWN_NMAX overrides.
int pick_down_nmax(int nmax_gu) {
    const int forced = [] {
        const int v = env_int("MOE_DOWN_NMAX", 0);
        return nmax_supported(v) ? v : 0;
    }();
    if (forced) return forced;
    return nmax_gu;
}

// 128-row weight sub-tiles per down-projection tile: two, i.e. one 3D copy of
// 32 KB of weights per pipeline stage against each token tile, which halves
// the token-tile re-reads (the down GEMM is bound by the bulk-copy rows it
// issues).  MOE_DOWN_MB overrides.
int pick_down_mb(int nmax) {
    const int forced = [] {
        const int v = env_int("MOE_DOWN_MB", 0);
        return (v == 1 || v == 2) ? v : 0;
    }();
    if (forced) return forced;
    (void)nmax;
    return 2;
}

// Router logits GEMM shape: the gate weight (E rows, one or two 128-row
// sub-tiles) against token chunks of 256 (32/64 for small batches).  With the
// problem's own workspace the K range is also split so that about one tile per
// SM runs (at most 8 parts): every CTA then reads only its part of the gate
// weight and of the chunk, instead of the whole 3 MB weight per 32 tokens.
// The parts land in separate fp32 slices that the top-k kernel sums in a fixed
// order.  The split depends only on the problem, so the workspace size does too.
constexpr int64_t kSplitTargetTiles = 148;  // SMs of a B200
struct LogitsPlan {
    int nmax, mb, splits;
};
LogitsPlan logits_plan(const moe_problem* p, bool allow_split) {
    LogitsPlan lp;
    lp.mb = p->E > 128 ? 2 : 1;
    lp.nmax = p->T >= 256 ? 256 : (p->T > 32 ? 64 : 32);
    lp.splits = 1;
    if (allow_split && p->dtype == MOE_BF16) {
        const int64_t chunks = (p->T + lp.nmax - 1) / lp.nmax;
        const int64_t nblk = (p->E + 128 * lp.mb - 1) / (128 * lp.mb);
        const int64_t base = std::max<int64_t>(1, chunks * nblk);
        const int64_t sp = std::min<int64_t>(kSplitTargetTiles / base, std::min<int64_t>(8, p->H / 64));
        lp.splits = static_cast<int>(std::max<int64_t>(1, sp));
    }
    return lp;
}


// Token chunks of the router GEMM (one routing counter each).
int64_t logits_chunks(const moe_problem* p) {
    const LogitsPlan lp = logits_plan(p, true);
    return std::max<int64_t>(1, (p->T + lp.nmax - 1) / lp.nmax);
}

// ------------------------------------------------------------------ workspace layout

struct Carve {
    size_t off = 0;
    size_t take(size_t bytes) {
        size_t o = off;
        off += (bytes + 255) & ~size_t(255);
        return o;
    }
};

struct Layout {
    size_t status, logits, rcount, idx, w, hist, base, counts, offsets, partial, sched_gu, sched_dn,
        pos, src, row_w;
    size_t x_perm, h_perm, out_acc, y_perm, x_q, s_x, total;
};

int64_t perm_chunks(int64_t T) { return (T + kPermTokens - 1) / kPermTokens; }
size_t sched_bytes() { return 5 * (kMaxSegments + 1) * sizeof(int32_t); }

Layout layout_for(const moe_problem* p, int call, int64_t ffn_rows = 0, int ffn_groups = 0) {
    Layout L{};
    Carve c;
    const int64_t T = p->T, H = p->H, E = p->E, I = p->I, k = p->top_k, S = p->num_shared;
    const bool f32 = p->dtype == MOE_F32;
    L.status = c.take(256);
    switch (call) {
        case MOE_CALL_ROUTER_LOGITS:
            break;
        case MOE_CALL_ROUTE:
            L.logits = c.take(logits_plan(p, true).splits * T * E * 4);
            L.rcount = c.take(logits_chunks(p) * 4);
            break;
        case MOE_CALL_PERMUTE:
            L.hist = c.take(perm_chunks(T) * E * 4);
            L.base = c.take(perm_chunks(T) * E * 4);
            L.counts = c.take(E * 4);
            break;
        case MOE_CALL_FFN:
            L.sched_gu = c.take(sched_bytes());
            L.sched_dn = c.take(sched_bytes());
            // fp32 problems keep h in fp32 (TF32 operand of the down GEMM)
            L.h_perm = c.take(ffn_rows * I * (f32 ? 4 : 2));
            break;
        case MOE_CALL_COMBINE:
            break;
        case MOE_CALL_ROUTER_STATS:
            L.logits = c.take(logits_plan(p, true).splits * T * E * 4);
            L.rcount = c.take(logits_chunks(p) * 4);
            L.idx = c.take(T * k * 4);
            L.w = c.take(T * k * 4);
            L.partial = c.take(((T + kStatsTokensPerBlock - 1) / kStatsTokensPerBlock) * E * 4);
            L.counts = c.take(E * 4);
            break;
        case MOE_CALL_FORWARD_FP8:
            L.logits = c.take(logits_plan(p, true).splits * T * E * 4);
            L.rcount = c.take(logits_chunks(p) * 4);
            L.idx = c.take(T * k * 4);
            L.w = c.take(T * k * 4);
            L.hist = c.take(perm_chunks(T) * E * 4);
            L.base = c.take(perm_chunks(T) * E * 4);
            L.counts = c.take(E * 4);
            L.offsets = c.take((E + 1) * 4);
            L.sched_gu = c.take(sched_bytes());
            L.sched_dn = c.take(sched_bytes());
            L.pos = c.take(T * k * 4);
            L.src = c.take(T * k * 4);
            L.row_w = c.take(T * k * 4);
            L.x_q = c.take(T * H);
            L.s_x = c.take(T * 4);
            L.x_perm = c.take(T * k * H);
            L.h_perm = c.take(T * (k + S) * I);
            L.y_perm = c.take(T * (k + S) * H * 2);
            break;
        case MOE_CALL_FORWARD:
        default:
            L.logits = c.take(logits_plan(p, true).splits * T * E * 4);
            L.rcount = c.take(logits_chunks(p) * 4);
            L.idx = c.take(T * k * 4);
            L.w = c.take(T * k * 4);
            L.hist = c.take(perm_chunks(T) * E * 4);
            L.base = c.take(perm_chunks(T) * E * 4);
            L.counts = c.take(E * 4);
            L.offsets = c.take((E + 1) * 4);
            L.sched_gu = c.take(sched_bytes());
            L.sched_dn = c.take(sched_bytes());
            L.pos = c.take(T * k * 4);
            L.src = c.take(T * k * 4);
            L.row_w = c.take(T * k * 4);
            // (fp32 problems: the permuted rows, h and the weighted rows in
            // fp32, the operands and results of the TF32 GEMMs)
            L.x_perm = c.take(T * k * H * (f32 ? 4 : 2));
            L.h_perm = c.take(T * (k + S) * I * (f32 ? 4 : 2));
            // weighted expert rows (gather combine) or the fp32 token
            // accumulator (scatter-add combine) share one region
            L.out_acc = c.take(std::max(T * (k + S) * H * (f32 ? 4 : 2), T * H * 4));
            L.y_perm = L.out_acc;
            break;
    }
    L.total = c.off;
    return L;
}

template <typename T>
T* at(void* ws, size_t off) {
    return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off);
}

// ------------------------------------------------------------------ GEMM launch

// Kernel launch on stream s; with pdl the launch may begin before the
// previous launch on the stream has finished (programmatic stream
// serialization): the kernel must then wait (griddepcontrol.wait) before it
// reads anything the previous launch writes.
template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*kern)(KArgs...), int grid, int threads, int smem, cudaStream_t s,
                      bool pdl, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(static_cast<unsigned>(threads));
    cfg.dynamicSmemBytes = static_cast<size_t>(smem);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Clusters of two CTAs (one per SM) of `kern` that can be resident at once.
template <typename K>
int resident_pairs(K kern, int threads, int smem) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) {
        cudaGetLastError();
        return 0;
    }
    return n;
}

template <int EPI, int NMAX, int MB, int ET = 0, bool PAIR = false, int GW = 0>
int32_t launch_gemm_n(const GemmArgs& a, int grid, cudaStream_t s, const char* name,
                      bool coop = false, bool pdl = false) {
    using C = GemmCfg<EPI, NMAX, MB, ET, PAIR, GW>;
    auto kern = grouped_gemm_kernel<EPI, NMAX, MB, ET, PAIR, GW>;
    int dev = 0;
    cudaGetDevice(&dev);
    static std::atomic<uint64_t> configured{0};
    static std::atomic<int> pairs[64];
    const uint64_t bit = (dev < 64) ? (1ull << dev) : 0;
    if (!bit || !(configured.load() & bit)) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::kSmemBytes) != cudaSuccess)
            return MOE_ERR_CUDA;
        if constexpr (PAIR) {
            const int n = resident_pairs(kern, C::kThreads, C::kSmemBytes);
            if (n < 1) return MOE_ERR_CUDA;
            if (bit) pairs[dev].store(n);
        }
        configured.fetch_or(bit);
    }
    if constexpr (PAIR) {
        // one cluster per pair tile (a tile = two adjacent CTA tiles), at most
        // as many clusters as can be resident together (persistent grid)
        const int n = bit ? pairs[dev].load() : resident_pairs(kern, C::kThreads, C::kSmemBytes);
        if (n < 1) return MOE_ERR_CUDA;
        const int clusters = std::max(1, std::min(n, (grid + 1) / 2));
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * clusters);
        cfg.blockDim = dim3(C::kThreads);
        cfg.dynamicSmemBytes = C::kSmemBytes;
        cfg.stream = s;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = pdl ? 2 : 1;
        MOE_LAUNCH(name, s, if (cudaLaunchKernelEx(&cfg, kern, a) != cudaSuccess) return MOE_ERR_CUDA);
    } else if (coop) {
        // every CTA resident at once (the fused routing phase waits across CTAs)
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(grid);
        cfg.blockDim = dim3(C::kThreads);
        cfg.dynamicSmemBytes = C::kSmemBytes;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        MOE_LAUNCH(name, s, if (cudaLaunchKernelEx(&cfg, kern, a) != cudaSuccess) return MOE_ERR_CUDA);
    } else {
        MOE_LAUNCH(name, s, if (launch_ex(kern, grid, C::kThreads, C::kSmemBytes, s, pdl, a) !=
                                cudaSuccess) return MOE_ERR_CUDA);
    }
    return MOE_OK;
}

// MOE_PAIR=1 runs the expert GEMMs as CTA pairs (cta_group::2, M = 256 per
// MMA, each CTA loading half of the token tile) for tiles of 64 or more token
// rows.  Off by default: the pairs halve the token-tile reads from L2 but
// measured slower at the Hy4 prefill shapes (the two CTAs advance in
// lockstep), and only about 1% faster on the tensor-bound skewed batch.
// Warps that gather the gate/up GEMM's token rows (the fused row gather).
// Three measured 1-3% faster per prefill layer than four (bf16 and FP8; Hy3
// 1%; decode unchanged) and two slower: with fewer warps, fewer of them
// compete with the epilogue for the shared-memory pipe, while three still keep
// the token-row stages ahead of the MMAs.
constexpr int kGatherWarps = 3;

bool use_pair() {
    const bool v = env_int("MOE_PAIR", 0) != 0;
    return v;
}

template <int EPI, int MB, int ET = 0>
int32_t launch_gemm_mb(int nmax, const GemmArgs& a, int grid, cudaStream_t s, const char* name,
                       bool pair = false, bool pdl = false) {
    switch (nmax) {
        case 16: return launch_gemm_n<EPI, 16, MB, ET>(a, grid, s, name, false, pdl);
        case 32: return launch_gemm_n<EPI, 32, MB, ET>(a, grid, s, name, false, pdl);
        case 64:
            return pair ? launch_gemm_n<EPI, 64, MB, ET, true>(a, grid, s, name, false, pdl)
                        : launch_gemm_n<EPI, 64, MB, ET>(a, grid, s, name, false, pdl);
        case 128:
            return pair ? launch_gemm_n<EPI, 128, MB, ET, true>(a, grid, s, name, false, pdl)
                        : launch_gemm_n<EPI, 128, MB, ET>(a, grid, s, name, false, pdl);
        case 160:
            return pair ? launch_gemm_n<EPI, 160, MB, ET, true>(a, grid, s, name, false, pdl)
                        : launch_gemm_n<EPI, 160, MB, ET>(a, grid, s, name, false, pdl);
        case 256:
            return pair ? launch_gemm_n<EPI, 256, MB, ET, true>(a, grid, s, name, false, pdl)
                        : launch_gemm_n<EPI, 256, MB, ET>(a, grid, s, name, false, pdl);
        default: return MOE_ERR_UNSUPPORTED;
    }
}

// FP8 expert GEMMs: gate/up (+SwiGLU) and down with the store epilogue.
template <int EPI>
int32_t launch_gemm_fp8(int nmax, int mb, const GemmArgs& a, int64_t max_tiles, cudaStream_t s,
                        const char* name, bool pdl = false) {
    int grid = static_cast<int>(std::min<int64_t>(sm_count(), std::max<int64_t>(1, max_tiles)));
    const bool pair = use_pair() && nmax >= 64;
    if constexpr (EPI == EPI_SWIGLU) {
        if (a.gather_tok != nullptr) {
            // E4M3 token rows gathered by the gather warps
            switch (nmax) {
                case 16: return launch_gemm_n<EPI, 16, 2, 1, false, kGatherWarps>(a, grid, s, name, false, pdl);
                case 32: return launch_gemm_n<EPI, 32, 2, 1, false, kGatherWarps>(a, grid, s, name, false, pdl);
                case 64: return launch_gemm_n<EPI, 64, 2, 1, false, kGatherWarps>(a, grid, s, name, false, pdl);
                case 128: return launch_gemm_n<EPI, 128, 2, 1, false, kGatherWarps>(a, grid, s, name, false, pdl);
                case 160: return launch_gemm_n<EPI, 160, 2, 1, false, kGatherWarps>(a, grid, s, name, false, pdl);
                case 256: return launch_gemm_n<EPI, 256, 2, 1, false, kGatherWarps>(a, grid, s, name, false, pdl);
                default: return MOE_ERR_UNSUPPORTED;
            }
        }
        return launch_gemm_mb<EPI, 2, 1>(nmax, a, grid, s, name, pair, pdl);
    } else {
        static_assert(EPI == EPI_DOWN_STORE, "FP8 down GEMM uses the store epilogue");
        if (mb == 2) return launch_gemm_mb<EPI, 2, 1>(nmax, a, grid, s, name, pair, pdl);
        return launch_gemm_mb<EPI, 1, 1>(nmax, a, grid, s, name, false, pdl);
    }
}

// TF32 expert GEMMs on fp32 operands (fp32 problems): gate/up (+SwiGLU, fp32
// h) and down (store or scatter-add epilogue), one CTA per tile.
template <int EPI>
int32_t launch_gemm_tf32(int nmax, int mb, const GemmArgs& a, int64_t max_tiles, cudaStream_t s,
                         const char* name, bool pdl = false) {
    int grid = static_cast<int>(std::min<int64_t>(sm_count(), std::max<int64_t>(1, max_tiles)));
    if constexpr (EPI == EPI_SWIGLU) {
        return launch_gemm_mb<EPI, 2, 2>(nmax, a, grid, s, name, false, pdl);
    } else {
        if (mb == 2) return launch_gemm_mb<EPI, 2, 2>(nmax, a, grid, s, name, false, pdl);
        return launch_gemm_mb<EPI, 1, 2>(nmax, a, grid, s, name, false, pdl);
    }
}

// Launch with a persistent grid of min(#SMs, tiles) CTAs.
template <int EPI>
int32_t launch_gemm(int nmax, int mb, const GemmArgs& a, int64_t max_tiles, cudaStream_t s,
                    const char* name, bool pdl = false) {
    int grid = static_cast<int>(std::min<int64_t>(sm_count(), std::max<int64_t>(1, max_tiles)));
    if constexpr (EPI == EPI_SWIGLU) {
        if (a.gather_tok != nullptr) {
            // row gather by the dedicated gather warps
            switch (nmax) {
                case 16: return launch_gemm_n<EPI, 16, 2, 0, false, kGatherWarps>(a, grid, s, name, false, pdl);
                case 32: return launch_gemm_n<EPI, 32, 2, 0, false, kGatherWarps>(a, grid, s, name, false, pdl);
                case 64: return launch_gemm_n<EPI, 64, 2, 0, false, kGatherWarps>(a, grid, s, name, false, pdl);
                case 128: return launch_gemm_n<EPI, 128, 2, 0, false, kGatherWarps>(a, grid, s, name, false, pdl);
                case 160: return launch_gemm_n<EPI, 160, 2, 0, false, kGatherWarps>(a, grid, s, name, false, pdl);
                case 256: return launch_gemm_n<EPI, 256, 2, 0, false, kGatherWarps>(a, grid, s, name, false, pdl);
                default: return MOE_ERR_UNSUPPORTED;
            }
        }
        const bool pair = use_pair() && nmax >= 64;
        return launch_gemm_mb<EPI, 2>(nmax, a, grid, s, name, pair, pdl);
    } else if constexpr (EPI == EPI_LOGITS) {
        if (nmax == 256) {
            if (mb == 2) return launch_gemm_n<EPI, 256, 2>(a, grid, s, name);
            return launch_gemm_n<EPI, 256, 1>(a, grid, s, name);
        }
        if (nmax == 64) {
            if (mb == 2) return launch_gemm_n<EPI, 64, 2>(a, grid, s, name);
            return launch_gemm_n<EPI, 64, 1>(a, grid, s, name);
        }
        if (nmax != 32) return MOE_ERR_UNSUPPORTED;
        if (mb == 2) return launch_gemm_n<EPI, 32, 2>(a, grid, s, name);
        return launch_gemm_n<EPI, 32, 1>(a, grid, s, name);
    } else {
        const bool pair = EPI == EPI_DOWN_STORE && use_pair() && nmax >= 64 && mb == 2;
        if (mb == 2) return launch_gemm_mb<EPI, 2>(nmax, a, grid, s, name, pair, pdl);
        return launch_gemm_mb<EPI, 1>(nmax, a, grid, s, name, false, pdl);
    }
}

// Upper bound on tiles of a schedule: sum over segments of ceil(rows/nmax)
// <= rows_total/nmax + nseg, times weight blocks of rows_per_tile rows.
int64_t max_tiles(int64_t rows_total, int nseg, int nmax, int64_t m_total,
                  int64_t rows_per_tile = 128) {
    return (rows_total / nmax + nseg) * ((m_total + rows_per_tile - 1) / rows_per_tile);
}

// How the expert rows are combined into token order (MOE_COMBINE=atomic picks
// the fp32 scatter-add in the down GEMM's epilogue).  Default: the down
// epilogue stores weighted bf16 rows and a gather kernel sums each token's
// rows in slot order, which is deterministic and leaves the L2 atomic units
// out of the critical path.
bool combine_atomic() {
    const bool v = [] {
        const char* e = std::getenv("MOE_COMBINE");
        return e && std::strcmp(e, "atomic") == 0;
    }();
    return v;
}

// Whether the gate/up GEMM gathers the routed token rows straight from x
// (kGatherWarps gather warps, 16-byte cp.async into the swizzled stage; bf16 rows,
// or the E4M3 code rows of moe_forward_fp8) instead of reading a permuted copy
// x_perm written by a separate
// gather kernel.  Default: fused for token tiles of up to 160 rows (measured
// 0.2-2% faster per layer at the Hy4 prefill and decode and the Hy3 batches,
// from dropping the gather launch and the copy's DRAM round trip), the
// permuted copy for wider tiles (the 256-row tiles of the skewed batch, where
// the gather warps slowed the tensor-bound GEMM by 10%).  MOE_FUSED_GATHER=0/1
// forces either form.
bool fused_gather(int nmax) {
    const int v = env_int("MOE_FUSED_GATHER", -1);
    if (v == 0 || v == 1) return v == 1;
    return nmax <= 160;
}

// L2 cache hints on the GEMM operand loads (MOE_L2_HINTS=0 turns them off).
int l2_hints() {
    const int v = env_int("MOE_L2_HINTS", 1) ? 1 : 0;
    return v;
}

// Rotated K order in the expert GEMMs (MOE_KROT=1; off by default):
// concurrent tiles start their K loops at different offsets instead of
// sweeping one column band of many rows in lockstep.  Measured 1.5% slower at
// the Hy4 prefill batch and 4% slower at the skewed one (the DRAM channels
// were already evenly loaded), so the plain order is the default.
int k_rotate() {
    const int v = env_int("MOE_KROT", 0) ? 1 : 0;
    return v;
}

// Programmatic dependent launch along the forward's kernel chain (MOE_PDL=0
// turns it off): each kernel may start while its predecessor finishes, does
// its independent set-up (in the expert GEMMs: streams its first weight
// tiles), then waits for the predecessor before reading its outputs.
bool pdl_enabled() {
    const bool v = env_int("MOE_PDL", 1) != 0;
    return v;
}

GemmArgs base_args(int32_t* status) {
    GemmArgs a;
    std::memset(&a, 0, sizeof(a));
    a.special_seg = -1;
    a.clip = INFINITY;
    a.l2_hints = l2_hints();
    a.status = status;
    return a;
}

// L2 policy of the weights of an expert cut into several token chunks
// (MOE_MULTI_CHUNK_L2: 0 evict-first, 1 normal (default), 2 evict-last).
// With evict-first, the skewed batch's heavy experts had their weights
// re-read from DRAM by almost every chunk (gate/up 29.4 GB of DRAM reads for
// 9.8 GB of weights and token rows); evict-normal keeps them in L2 across the
// chunks that run together (13.5 GB) and measured the fastest of the three.
int multi_chunk_policy() {
    const int v = env_int("MOE_MULTI_CHUNK_L2", 1);
    return (v >= 0 && v <= 2) ? v : 1;
}

// Expert GEMM arguments: K order, the multi-chunk weight policy, and whether
// the following launch may start as soon as this one has passed its
// dependency wait.
void expert_gemm_launch_args(GemmArgs& a, bool trigger_early) {
    a.k_rotate = k_rotate();
    a.multi_chunk_policy = multi_chunk_policy();
    a.pdl_trigger_early = trigger_early ? 1 : 0;
}

// Fused routing outputs of the router GEMM (see GemmArgs::route_idx).
struct RouteOut {
    const float* bias;
    int32_t* idx;
    float* w;
    int32_t* count;  // logits_chunks(p) counters, zeroed here
    bool keep_sum;
};

constexpr int kFusedRouteMaxTokens = 32;  // tokens one CTA routes in the fused launch

// MOE_FUSED_ROUTE=0 keeps the router GEMM and the top-k kernel separate.
bool fused_route_enabled() {
    const bool v = env_int("MOE_FUSED_ROUTE", 1) != 0;
    return v;
}

// Router logits through tcgen05 (bf16 x and gate weight); with `route`, the
// same launch also routes every token (one tile per CTA, cooperative launch).
int32_t run_logits_bf16(const moe_problem* p, const void* x, const void* gate_w, float* logits,
                        int32_t* status, cudaStream_t s, const LogitsPlan& lp,
                        const RouteOut* route = nullptr) {
    GemmArgs a = base_args(status);
    if (!make_tmap(&a.tmA0, gate_w, p->E, p->H, 128 * lp.mb)) return MOE_ERR_CUDA;
    if (!make_tmap_rows(a.tmB0, x, p->T, p->H)) return MOE_ERR_CUDA;
    a.tmA1 = a.tmA0;
    for (int j = 0; j < kNumBoxSizes; ++j) a.tmB1[j] = a.tmB0[j];
    a.sched = nullptr;
    a.single_rows = static_cast<int32_t>(p->T);
    a.single_chunk_len = lp.nmax;
    a.nseg = 1;
    a.K = p->H;
    a.M_total = p->E;
    a.out = logits;
    a.out_ld = p->E;
    a.k_splits = lp.splits;
    a.split_stride = p->T * static_cast<int64_t>(p->E);
    if (route) {
        const int64_t chunks = (p->T + lp.nmax - 1) / lp.nmax;
        const int64_t tiles = chunks * lp.splits;  // one weight block: E <= 128 * mb
        if (cudaMemsetAsync(route->count, 0, chunks * sizeof(int32_t), s) != cudaSuccess)
            return MOE_ERR_CUDA;
        a.route_idx = route->idx;
        a.route_w = route->w;
        a.route_bias = route->bias;
        a.route_count = route->count;
        a.route_k = p->top_k;
        a.route_scale = p->routed_scale;
        a.route_keep_sum = route->keep_sum ? 1 : 0;
        const int grid = static_cast<int>(tiles);
        const char* name = "router_gemm_topk";
        if (lp.nmax == 256) {
            if (lp.mb == 2) return launch_gemm_n<EPI_LOGITS, 256, 2>(a, grid, s, name, true);
            return launch_gemm_n<EPI_LOGITS, 256, 1>(a, grid, s, name, true);
        }
        if (lp.nmax == 64) {
            if (lp.mb == 2) return launch_gemm_n<EPI_LOGITS, 64, 2>(a, grid, s, name, true);
            return launch_gemm_n<EPI_LOGITS, 64, 1>(a, grid, s, name, true);
        }
        if (lp.mb == 2) return launch_gemm_n<EPI_LOGITS, 32, 2>(a, grid, s, name, true);
        return launch_gemm_n<EPI_LOGITS, 32, 1>(a, grid, s, name, true);
    }
    return launch_gemm<EPI_LOGITS>(
        lp.nmax, lp.mb, a, max_tiles(p->T, 1, lp.nmax, p->E, 128 * lp.mb) * lp.splits, s,
        "router_logits_gemm");
}

// Router logits into `logits`; with split = true (the problem's own workspace)
// the K parts go to consecutive [T,E] slices (logits_plan(p, true).splits of
// them) for run_topk to sum.
int32_t run_logits(const moe_problem* p, const void* x, const void* gate_w, float* logits,
                   int32_t* status, cudaStream_t s, bool split = false) {
    if (p->dtype == MOE_BF16)
        return run_logits_bf16(p, x, gate_w, logits, status, s, logits_plan(p, split));
    MOE_LAUNCH("router_logits_f32", s,
               router_logits_f32_kernel<<<static_cast<unsigned>(p->T), 256, 0, s>>>(
                   static_cast<const float*>(x), static_cast<const float*>(gate_w), p->H, p->E,
                   logits));
    return MOE_OK;
}

// Top-k over the logits; n_parts > 1 sums that many [T,E] slices first (in
// slice order), leaving the sum in the first slice when keep_sum is set.
int32_t run_topk(const moe_problem* p, float* logits, const float* bias, int32_t* idx, float* w,
                 cudaStream_t s, int n_parts = 1, bool keep_sum = false) {
    const int warps = 8;
    const unsigned blocks = static_cast<unsigned>((p->T + warps - 1) / warps);
    MOE_LAUNCH("route_topk", s,
               topk_kernel<<<blocks, warps * 32, 0, s>>>(logits, n_parts, p->T * p->E, keep_sum,
                                                         bias, p->T, p->E, p->top_k,
                                                         p->routed_scale, idx, w));
    return MOE_OK;
}

// Routing for the problem's own workspace: the fused router GEMM + top-k
// launch (bf16, at most one tile per SM), else the K-split router GEMM and
// the top-k kernel.  logits: logits_plan(p, true).splits [T,E] slices;
// count: logits_chunks(p) ints.
int32_t run_route(const moe_problem* p, const void* x, const void* gate_w, const float* bias,
                  float* logits, int32_t* count, int32_t* idx, float* w, bool keep_sum,
                  int32_t* status, cudaStream_t s) {
    const LogitsPlan lp = logits_plan(p, true);
    // fused when every tile has its own SM and each CTA routes at most 32
    // tokens afterwards (at 128 per CTA the two launches measured faster)
    const int per_cta = (lp.nmax + lp.splits - 1) / lp.splits;
    if (p->dtype == MOE_BF16 && fused_route_enabled() &&
        logits_chunks(p) * lp.splits <= sm_count() && per_cta <= kFusedRouteMaxTokens) {
        const RouteOut r{bias, idx, w, count, keep_sum};
        return run_logits_bf16(p, x, gate_w, logits, status, s, lp, &r);
    }
    const int32_t rc = run_logits(p, x, gate_w, logits, status, s, true);
    if (rc != MOE_OK) return rc;
    return run_topk(p, logits, bias, idx, w, s, lp.splits, keep_sum);
}


template <typename TIn, typename TOut>
int32_t run_gather(const TIn* x, int64_t T, int H, int k, const int32_t* pos, int64_t n_rows,
                   TOut* x_perm, __nv_bfloat16* x_bf16, float* acc_zero, cudaStream_t s,
                   bool pdl = false);

}  // namespace

// Copy each token row into its k permuted rows (optionally converting), one
// warp per token.  Also writes a bf16 copy of x and zeroes the token's fp32
// accumulator row when asked.
template <typename TIn, typename TOut>
__global__ void gather_kernel(const TIn* __restrict__ x, int64_t T, int H, int k,
                              const int32_t* __restrict__ pos, int64_t n_rows,
                              TOut* __restrict__ x_perm, __nv_bfloat16* __restrict__ x_bf16,
                              float* __restrict__ acc_zero) {
    // one warp per (token, segment of 32 * kBatch output vectors)
    constexpr int kElems0 = 16 / sizeof(TOut);
    constexpr int kSeg = 32 * 8;
    const int lane = threadIdx.x & 31;
    const int nseg = (H / kElems0 + kSeg - 1) / kSeg;
    const int64_t gw = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int64_t t = gw / nseg;
    if (t >= T) return;
    const int seg = static_cast<int>(gw - t * nseg);
    ptx::grid_dep_wait();  // positions come from the previous launch
    ptx::grid_dep_launch();
    int my_pos = -1;
    if (lane < k) {
        my_pos = pos[t * k + lane];
        if (my_pos < 0 || my_pos >= n_rows) my_pos = -1;
    }
    constexpr int kElems = 16 / sizeof(TOut);  // elements per 16-byte output vector
    constexpr int kBatch = 8;  // 16-byte loads in flight per lane before the stores
    static_assert(32 * kBatch == kSeg, "segment = one batch");
    const int nvec = H / kElems;
    {
        const int v0 = seg * kSeg;
        uint4 packed[kBatch];
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            const int v = v0 + b * 32 + lane;
            if (v < nvec) {
                if constexpr (sizeof(TIn) == sizeof(TOut)) {
                    packed[b] = reinterpret_cast<const uint4*>(x + t * H)[v];
                } else {
                    // fp32 -> bf16: 8 inputs per output vector
                    const float4 a = reinterpret_cast<const float4*>(x + t * H)[2 * v];
                    const float4 c = reinterpret_cast<const float4*>(x + t * H)[2 * v + 1];
                    __nv_bfloat162 p0 = __floats2bfloat162_rn(a.x, a.y);
                    __nv_bfloat162 p1 = __floats2bfloat162_rn(a.z, a.w);
                    __nv_bfloat162 p2 = __floats2bfloat162_rn(c.x, c.y);
                    __nv_bfloat162 p3 = __floats2bfloat162_rn(c.z, c.w);
                    packed[b].x = *reinterpret_cast<uint32_t*>(&p0);
                    packed[b].y = *reinterpret_cast<uint32_t*>(&p1);
                    packed[b].z = *reinterpret_cast<uint32_t*>(&p2);
                    packed[b].w = *reinterpret_cast<uint32_t*>(&p3);
                }
            }
        }
#pragma unroll
        for (int b = 0; b < kBatch; ++b) {
            const int v = v0 + b * 32 + lane;
            const bool ok = v < nvec;
            if constexpr (sizeof(TIn) != sizeof(TOut)) {
                if (ok && x_bf16) reinterpret_cast<uint4*>(x_bf16 + t * H)[v] = packed[b];
            }
            // every lane takes part in the shuffles; only the stores are predicated
            for (int j = 0; j < k; ++j) {
                const int r = __shfl_sync(0xffffffffu, my_pos, j);
                if (ok && r >= 0)
                    reinterpret_cast<uint4*>(x_perm + static_cast<int64_t>(r) * H)[v] = packed[b];
            }
        }
    }
    if (acc_zero) {
        // this segment's share of the token's fp32 accumulator row
        const int per = (H / 4 + nseg - 1) / nseg;
        float4* z = reinterpret_cast<float4*>(acc_zero + t * H);
        for (int v = seg * per + lane; v < min(H / 4, (seg + 1) * per); v += 32)
            z[v] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

namespace {

template <typename TIn, typename TOut>
int32_t run_gather(const TIn* x, int64_t T, int H, int k, const int32_t* pos, int64_t n_rows,
                   TOut* x_perm, __nv_bfloat16* x_bf16, float* acc_zero, cudaStream_t s,
                   bool pdl) {
    const int warps = 8;
    const int64_t segs = (H / (16 / static_cast<int>(sizeof(TOut))) + 32 * 8 - 1) / (32 * 8);
    const int blocks = static_cast<int>((T * segs + warps - 1) / warps);
    MOE_LAUNCH("dispatch_gather", s,
               if (launch_ex(gather_kernel<TIn, TOut>, blocks, warps * 32, 0, s, pdl, x, T, H, k,
                             pos, n_rows, x_perm, x_bf16, acc_zero) != cudaSuccess)
                   return MOE_ERR_CUDA);
    return MOE_OK;
}

// out[t] = sum over the token's rows of y (slot order, the shared row last),
// one warp per (token, segment of H).
template <typename TIn, typename TOut>
int32_t run_gather_sum(const TIn* y, const int32_t* pos, int64_t T, int H, int k,
                       int64_t n_rows, int64_t shared_row0, TOut* out, int32_t* status,
                       cudaStream_t s, bool pdl = false) {
    // three rows' loads in flight, two 16-byte vectors per lane and row (1 KB
    // segments of H per warp): measured 9-10% faster than two rows, and faster
    // than more rows or more (or fewer) vectors per lane, whose segments or
    // register use cost more than the extra loads in flight gain
    constexpr int kBatch = 3, kVPL = 2;
    const int warps = 8;
    const int vec = 16 / static_cast<int>(sizeof(TIn));
    const int64_t segs = (H / vec + 32 * kVPL - 1) / (32 * kVPL);
    const int blocks = static_cast<int>((T * segs + warps - 1) / warps);
    MOE_LAUNCH("combine_gather", s,
               if (launch_ex(gather_sum_kernel<TIn, TOut, kBatch, kVPL>, blocks, warps * 32, 0, s,
                             pdl, y, pos, T, H, k, n_rows, shared_row0, out, status) !=
                   cudaSuccess) return MOE_ERR_CUDA);
    return MOE_OK;
}

// histogram -> scan (+ schedules) -> stable scatter
int32_t run_dispatch(const moe_problem* p, const int32_t* idx, const float* topk_w, int32_t* hist,
                     int32_t* base, int32_t* counts, int32_t* offsets, int32_t* sched_gu,
                     int nmax_gu, int32_t* sched_dn, int nmax_dn, int32_t* pos, int32_t* src,
                     float* row_w, int32_t* status, cudaStream_t s) {
    const int nch = static_cast<int>(perm_chunks(p->T));
    const bool pdl = pdl_enabled();
    MOE_LAUNCH("dispatch_count", s,
               dispatch_count_kernel<<<nch, kPermTokens, 0, s>>>(idx, p->T, p->E, p->top_k, hist,
                                                                 status));
    MOE_LAUNCH("dispatch_scan", s,
               if (launch_ex(dispatch_scan_kernel, 1, 512, 0, s, pdl, hist, nch, p->E, p->T,
                             p->top_k, p->num_shared, base, counts, offsets, sched_gu, nmax_gu,
                             sched_dn, nmax_dn) != cudaSuccess) return MOE_ERR_CUDA);
    MOE_LAUNCH("dispatch_scatter", s,
               if (launch_ex(dispatch_scatter_kernel, nch, kPermTokens, 0, s, pdl, idx, topk_w,
                             p->T, p->E, p->top_k, base, offsets, pos, src, row_w, status) !=
                   cudaSuccess) return MOE_ERR_CUDA);
    return MOE_OK;
}

template <typename TOut>
int32_t run_finalize(const float* acc, TOut* out, int64_t n, cudaStream_t s, bool pdl = false) {
    const int64_t n4 = n / 4;
    const int blocks =
        static_cast<int>(std::max<int64_t>(1, std::min<int64_t>((n4 + 255) / 256, 148 * 8)));
    MOE_LAUNCH("finalize", s,
               if (launch_ex(finalize_kernel<TOut>, blocks, 256, 0, s, pdl, acc, out, n4) !=
                   cudaSuccess) return MOE_ERR_CUDA);
    return MOE_OK;
}

#define MOE_TRY(expr)                      \
    do {                                   \
        int32_t r_ = (expr);               \
        if (r_ != MOE_OK) return r_;       \
    } while (0)

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" {

const char* moe_status_string(int32_t status) {
    switch (status) {
        case MOE_OK: return "ok";
        case MOE_ERR_INVALID_ARG: return "invalid argument";
        case MOE_ERR_UNSUPPORTED: return "unsupported shape or dtype";
        case MOE_ERR_WORKSPACE: return "workspace missing or too small";
        case MOE_ERR_CUDA: return "CUDA launch or runtime error";
        case MOE_ERR_TIMEOUT: return "device wait timed out";
        case MOE_ERR_BAD_INDEX: return "index input out of range";
        default: return "unknown status";
    }
}

size_t moe_workspace_size(const moe_problem* p, int32_t call) {
    if (check_problem(p) != MOE_OK) return 0;
    if (call < MOE_CALL_ROUTE || call > MOE_CALL_FORWARD_FP8) return 0;
    if (call == MOE_CALL_FFN) {
        // the FFN workspace depends on rows/groups; size it for the routed
        // rows of this problem (T*top_k) and E groups, the larger of the two
        // uses (routed experts, or the shared expert over T rows)
        const int64_t rows = std::max<int64_t>(p->T * p->top_k, p->T);
        return layout_for(p, call, rows, p->E).total;
    }
    return layout_for(p, call).total;
}

int32_t moe_expert_tile_rows(const moe_problem* p, int32_t* gate_up_rows, int32_t* down_rows) {
    MOE_TRY(check_problem(p));
    if (!gate_up_rows || !down_rows) return MOE_ERR_INVALID_ARG;
    const int nmax = pick_nmax(static_cast<double>(p->T * p->top_k) / p->E);
    *gate_up_rows = nmax;
    *down_rows = pick_down_nmax(nmax);
    return MOE_OK;
}

int32_t moe_router_logits(const moe_problem* p, const void* x, const void* gate_w, float* logits,
                          void* ws, size_t ws_bytes, void* stream) {
    MOE_TRY(check_problem(p));
    if (!x || !gate_w || !logits || !ws) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(gate_w) || !aligned16(logits) || !aligned16(ws))
        return MOE_ERR_INVALID_ARG;
    if (ws_bytes < layout_for(p, MOE_CALL_ROUTER_LOGITS).total) return MOE_ERR_WORKSPACE;
    if (p->T == 0) return MOE_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    return run_logits(p, x, gate_w, logits, at<int32_t>(ws, 0), s);
}

int32_t moe_route(const moe_problem* p, const void* x, const void* gate_w, const float* bias,
                  int32_t* topk_idx, float* topk_w, void* ws, size_t ws_bytes, void* stream) {
    MOE_TRY(check_problem(p));
    if (!x || !gate_w || !topk_idx || !topk_w || !ws) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(gate_w) || !aligned16(ws)) return MOE_ERR_INVALID_ARG;
    const Layout L = layout_for(p, MOE_CALL_ROUTE);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
    if (p->T == 0) return MOE_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t* status = at<int32_t>(ws, L.status);
    float* logits = at<float>(ws, L.logits);
    return run_route(p, x, gate_w, bias, logits, at<int32_t>(ws, L.rcount), topk_idx, topk_w,
                     false, status, s);
}

int32_t moe_permute(const moe_problem* p, const int32_t* topk_idx, const void* x,
                    int32_t* offsets, int32_t* pos, int32_t* src_token, void* x_perm, void* ws,
                    size_t ws_bytes, void* stream) {
    MOE_TRY(check_problem(p));
    if (!topk_idx || !x || !offsets || !pos || !src_token || !x_perm || !ws)
        return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(x_perm) || !aligned16(ws)) return MOE_ERR_INVALID_ARG;
    const Layout L = layout_for(p, MOE_CALL_PERMUTE);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
    if (p->T == 0) {
        // offsets are all zero for an empty batch
        if (cudaMemsetAsync(offsets, 0, (p->E + 1) * sizeof(int32_t),
                            static_cast<cudaStream_t>(stream)) != cudaSuccess)
            return MOE_ERR_CUDA;
        return MOE_OK;
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t* status = at<int32_t>(ws, L.status);
    MOE_TRY(run_dispatch(p, topk_idx, nullptr, at<int32_t>(ws, L.hist), at<int32_t>(ws, L.base),
                         at<int32_t>(ws, L.counts), offsets, nullptr, 16, nullptr, 16, pos,
                         src_token, nullptr, status, s));
    const int64_t n_rows = p->T * p->top_k;
    if (p->dtype == MOE_BF16) {
        return run_gather<__nv_bfloat16, __nv_bfloat16>(
            static_cast<const __nv_bfloat16*>(x), p->T, p->H, p->top_k, pos, n_rows,
            static_cast<__nv_bfloat16*>(x_perm), nullptr, nullptr, s);
    }
    return run_gather<float, float>(static_cast<const float*>(x), p->T, p->H, p->top_k, pos,
                                    n_rows, static_cast<float*>(x_perm), nullptr, nullptr, s);
}

int32_t moe_grouped_swiglu_ffn(const moe_problem* p, const void* x_perm, int64_t rows,
                               const int32_t* offsets, int32_t n_groups, const void* expert_w,
                               void* y_perm, void* ws, size_t ws_bytes, void* stream) {
    MOE_TRY(check_problem(p));
    if (!x_perm || !offsets || !expert_w || !y_perm || !ws) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x_perm) || !aligned16(expert_w) || !aligned16(y_perm) || !aligned16(ws))
        return MOE_ERR_INVALID_ARG;
    if (n_groups < 1 || n_groups > kMaxExperts) return MOE_ERR_UNSUPPORTED;
    if (rows < 0 || rows >= (int64_t(1) << 31)) return MOE_ERR_UNSUPPORTED;
    if (static_cast<int64_t>(n_groups) * 3 * p->I >= (int64_t(1) << 31))
        return MOE_ERR_UNSUPPORTED;
    const Layout L = layout_for(p, MOE_CALL_FFN, rows, n_groups);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
    if (rows == 0) return MOE_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t* status = at<int32_t>(ws, L.status);
    const int64_t H = p->H, I = p->I;
    const void* xb = x_perm;
    const void* wb = expert_w;
    // fp32 problems: TF32 GEMMs on the fp32 operands as given
    const bool f32 = p->dtype == MOE_F32;
    const ElemType et = f32 ? kF32 : kBF16;
    const int nmax = pick_nmax(static_cast<double>(rows) / n_groups);
    int32_t* sg = at<int32_t>(ws, L.sched_gu);
    int32_t* sd = at<int32_t>(ws, L.sched_dn);
    MOE_LAUNCH("ffn_schedule", s,
               schedule_from_offsets_kernel<<<1, 32, 0, s>>>(offsets, n_groups, rows, sg, nmax, sd,
                                                             nmax, status));
    void* h = at<void>(ws, L.h_perm);
    {
        GemmArgs a = base_args(status);
        if (!make_tmap_gateup(&a.tmA0, wb, static_cast<int64_t>(n_groups) * 3, I, H, et))
            return MOE_ERR_CUDA;
        if (!make_tmap_rows(a.tmB0, xb, rows, H, et)) return MOE_ERR_CUDA;
        a.tmA1 = a.tmA0;
        for (int j = 0; j < kNumBoxSizes; ++j) a.tmB1[j] = a.tmB0[j];
        a.sched = sg;
        a.nseg = n_groups;
        a.K = static_cast<int32_t>(H);
        a.M_total = static_cast<int32_t>(I);
        a.a_seg_stride = 3;  // matrices per expert
        a.a_off0 = 0;
        a.out = h;
        a.out_ld = static_cast<int32_t>(I);
        a.clip = effective_clip(p);
        // an ordinary launch: the schedule it reads first is the previous
        // launch's output; the down GEMM may start as soon as it is resident
        expert_gemm_launch_args(a, true);
        if (f32)
            MOE_TRY(launch_gemm_tf32<EPI_SWIGLU>(nmax, 2, a, max_tiles(rows, n_groups, nmax, I), s,
                                                 "expert_gate_up_gemm_tf32"));
        else
            MOE_TRY(launch_gemm<EPI_SWIGLU>(nmax, 2, a, max_tiles(rows, n_groups, nmax, I), s,
                                            "expert_gate_up_gemm"));
    }
    {
        GemmArgs a = base_args(status);
        const int mb = pick_down_mb(nmax);
        if (!make_tmap_down(&a.tmA0, wb, static_cast<int64_t>(n_groups) * 3 * I, H, mb, et))
            return MOE_ERR_CUDA;
        if (!make_tmap_rows(a.tmB0, h, rows, I, et)) return MOE_ERR_CUDA;
        a.tmA1 = a.tmA0;
        for (int j = 0; j < kNumBoxSizes; ++j) a.tmB1[j] = a.tmB0[j];
        a.sched = sd;
        a.nseg = n_groups;
        a.K = static_cast<int32_t>(I);
        a.M_total = static_cast<int32_t>(H);
        a.a_seg_stride = static_cast<int32_t>(3 * I);
        a.a_off0 = static_cast<int32_t>(2 * I);
        a.out = y_perm;
        a.out_ld = static_cast<int32_t>(H);
        a.out_f32 = f32 ? 1 : 0;
        const bool pdl = pdl_enabled();
        expert_gemm_launch_args(a, false);
        if (f32)
            MOE_TRY(launch_gemm_tf32<EPI_DOWN_STORE>(nmax, mb, a,
                                                     max_tiles(rows, n_groups, nmax, H, 128 * mb),
                                                     s, "expert_down_gemm_tf32", pdl));
        else
            MOE_TRY(launch_gemm<EPI_DOWN_STORE>(nmax, mb, a,
                                                max_tiles(rows, n_groups, nmax, H, 128 * mb), s,
                                                "expert_down_gemm", pdl));
    }
    return MOE_OK;
}

int32_t moe_combine(const moe_problem* p, const void* y_perm, const int32_t* pos,
                    const float* topk_w, const void* shared_y, void* out, void* ws,
                    size_t ws_bytes, void* stream) {
    MOE_TRY(check_problem(p));
    if (!y_perm || !pos || !topk_w || !out || !ws) return MOE_ERR_INVALID_ARG;
    if (p->num_shared && !shared_y) return MOE_ERR_INVALID_ARG;
    const Layout L = layout_for(p, MOE_CALL_COMBINE);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
    if (p->T == 0) return MOE_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t* status = at<int32_t>(ws, L.status);
    const int64_t n_rows = p->T * p->top_k;
    const void* sy = p->num_shared ? shared_y : nullptr;
    const unsigned blocks = static_cast<unsigned>(p->T);
    if (p->dtype == MOE_BF16) {
        MOE_LAUNCH("combine", s,
                   combine_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(
                       static_cast<const __nv_bfloat16*>(y_perm), pos, topk_w,
                       static_cast<const __nv_bfloat16*>(sy), p->T, p->H, p->top_k, n_rows,
                       static_cast<__nv_bfloat16*>(out), status));
    } else {
        MOE_LAUNCH("combine", s,
                   combine_kernel<float><<<blocks, 256, 0, s>>>(
                       static_cast<const float*>(y_perm), pos, topk_w,
                       static_cast<const float*>(sy), p->T, p->H, p->top_k, n_rows,
                       static_cast<float*>(out), status));
    }
    return MOE_OK;
}

int32_t moe_forward(const moe_problem* p, const void* x, const void* gate_w, const float* bias,
                    const void* expert_w, const void* shared_w, void* out, int32_t* idx_out,
                    float* w_out, void* ws, size_t ws_bytes, void* stream) {
    MOE_TRY(check_problem(p));
    if (!x || !gate_w || !expert_w || !out || !ws) return MOE_ERR_INVALID_ARG;
    if (p->num_shared && !shared_w) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(gate_w) || !aligned16(expert_w) || !aligned16(out) ||
        !aligned16(ws) || (shared_w && !aligned16(shared_w)))
        return MOE_ERR_INVALID_ARG;
    const Layout L = layout_for(p, MOE_CALL_FORWARD);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
    if (p->T == 0) return MOE_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t* status = at<int32_t>(ws, L.status);
    const int64_t T = p->T, H = p->H, E = p->E, I = p->I, k = p->top_k, S = p->num_shared;
    const bool f32 = p->dtype == MOE_F32;

    int32_t* idx = idx_out ? idx_out : at<int32_t>(ws, L.idx);
    float* w = w_out ? w_out : at<float>(ws, L.w);
    float* logits = at<float>(ws, L.logits);

    // the tensor-core GEMMs read the weights as given: bf16 (kind::f16) or,
    // for fp32 problems, fp32 read as TF32 (kind::tf32)
    const void* ew = expert_w;
    const void* sw = shared_w;
    const ElemType et = f32 ? kF32 : kBF16;

    // 1. route
    MOE_TRY(run_route(p, x, gate_w, bias, logits, at<int32_t>(ws, L.rcount), idx, w, false,
                      status, s));

    // 2. dispatch bookkeeping + schedules
    const int nmax = pick_nmax(static_cast<double>(T * k) / E);
    const int nmax_dn = pick_down_nmax(nmax);
    int32_t* sg = at<int32_t>(ws, L.sched_gu);
    int32_t* sd = at<int32_t>(ws, L.sched_dn);
    int32_t* pos = at<int32_t>(ws, L.pos);
    int32_t* src = at<int32_t>(ws, L.src);
    float* row_w = at<float>(ws, L.row_w);
    MOE_TRY(run_dispatch(p, idx, w, at<int32_t>(ws, L.hist), at<int32_t>(ws, L.base),
                         at<int32_t>(ws, L.counts), at<int32_t>(ws, L.offsets), sg, nmax, sd,
                         nmax_dn, pos, src, row_w, status, s));

    // 3. token rows for the gate/up GEMM: gathered inside the GEMM (from x, by
    //    src) or copied into x_perm in expert order by the gather kernel (the
    //    problem dtype: fp32 rows for fp32 problems).  The scatter-add combine
    //    also needs its fp32 accumulator zeroed.
    void* x_perm = at<void>(ws, L.x_perm);
    // launches from here on may start while their predecessor finishes: each
    // waits for it before reading its outputs, and reads nothing earlier than
    // that except what was complete before the predecessor could start
    const bool pdl = pdl_enabled();
    const bool atomic_combine = combine_atomic();
    float* out_acc = atomic_combine ? at<float>(ws, L.out_acc) : nullptr;
    void* y_perm = at<void>(ws, L.y_perm);
    const bool gather_in_gemm = !f32 && fused_gather(nmax);
    if (f32) {
        MOE_TRY((run_gather<float, float>(static_cast<const float*>(x), T, p->H, p->top_k, pos,
                                          T * k, static_cast<float*>(x_perm), nullptr, out_acc, s,
                                          pdl)));
    } else if (!gather_in_gemm) {
        MOE_TRY((run_gather<__nv_bfloat16, __nv_bfloat16>(
            static_cast<const __nv_bfloat16*>(x), T, p->H, p->top_k, pos, T * k,
            static_cast<__nv_bfloat16*>(x_perm), nullptr, out_acc, s, pdl)));
    } else if (out_acc) {
        if (cudaMemsetAsync(out_acc, 0, static_cast<size_t>(T) * H * sizeof(float), s) !=
            cudaSuccess)
            return MOE_ERR_CUDA;
    }

    // 4. grouped gate/up GEMM + clamp + SwiGLU (routed experts, then shared)
    void* h = at<void>(ws, L.h_perm);
    const int64_t h_rows = T * (k + S);
    const int nseg = static_cast<int>(E + S);
    {
        GemmArgs a = base_args(status);
        if (!make_tmap_gateup(&a.tmA0, ew, E * 3, I, H, et)) return MOE_ERR_CUDA;
        if (!make_tmap_rows(a.tmB0, x_perm, T * k, H, et)) return MOE_ERR_CUDA;
        if (S) {
            if (!make_tmap_gateup(&a.tmA1, sw, 3, I, H, et)) return MOE_ERR_CUDA;
            if (!make_tmap_rows(a.tmB1, x, T, H, et)) return MOE_ERR_CUDA;
        } else {
            a.tmA1 = a.tmA0;
            for (int j = 0; j < kNumBoxSizes; ++j) a.tmB1[j] = a.tmB0[j];
        }
        a.sched = sg;
        a.nseg = nseg;
        a.special_seg = S ? static_cast<int32_t>(E) : -1;
        a.K = static_cast<int32_t>(H);
        a.M_total = static_cast<int32_t>(I);
        a.a_seg_stride = 3;  // matrices per expert
        a.a_off0 = 0;
        a.out = h;
        a.out_ld = static_cast<int32_t>(I);
        a.clip = effective_clip(p);
        if (gather_in_gemm) {
            a.gather_tok = src;
            a.gather_src = x;
            a.n_tokens = static_cast<int32_t>(T);
        }
        // (after a memset, the scatter-add mode's fused-gather form, the
        // launch is an ordinary one)
        const bool pdl_gu = pdl && !(gather_in_gemm && out_acc);
        expert_gemm_launch_args(a, true);
        if (f32)
            MOE_TRY(launch_gemm_tf32<EPI_SWIGLU>(nmax, 2, a, max_tiles(h_rows, nseg, nmax, I), s,
                                                 "expert_gate_up_gemm_tf32", pdl_gu));
        else
            MOE_TRY(launch_gemm<EPI_SWIGLU>(nmax, 2, a, max_tiles(h_rows, nseg, nmax, I), s,
                                            "expert_gate_up_gemm", pdl_gu));
    }
    // 5. grouped down GEMM; its epilogue applies the routing weight and either
    //    stores the weighted rows (gather combine) or scatter-adds them into the
    //    fp32 token accumulator
    {
        GemmArgs a = base_args(status);
        const int mb = pick_down_mb(nmax_dn);
        if (!make_tmap_down(&a.tmA0, ew, E * 3 * I, H, mb, et)) return MOE_ERR_CUDA;
        if (!make_tmap_rows(a.tmB0, h, h_rows, I, et)) return MOE_ERR_CUDA;
        if (S) {
            if (!make_tmap_down(&a.tmA1, sw, 3 * I, H, mb, et)) return MOE_ERR_CUDA;
        } else {
            a.tmA1 = a.tmA0;
        }
        for (int j = 0; j < kNumBoxSizes; ++j) a.tmB1[j] = a.tmB0[j];
        a.sched = sd;
        a.nseg = nseg;
        a.special_seg = S ? static_cast<int32_t>(E) : -1;
        a.K = static_cast<int32_t>(I);
        a.M_total = static_cast<int32_t>(H);
        a.a_seg_stride = static_cast<int32_t>(3 * I);
        a.a_off0 = static_cast<int32_t>(2 * I);
        a.out_ld = static_cast<int32_t>(H);
        a.n_tokens = static_cast<int32_t>(T);
        a.row_token = src;
        a.row_weight = row_w;
        a.routed_rows = static_cast<int32_t>(T * k);
        const int64_t tiles = max_tiles(h_rows, nseg, nmax_dn, H, 128 * mb);
        expert_gemm_launch_args(a, false);
        if (atomic_combine) {
            a.out = out_acc;
            if (f32)
                MOE_TRY(launch_gemm_tf32<EPI_DOWN_ATOMIC>(nmax_dn, mb, a, tiles, s,
                                                          "expert_down_combine_gemm_tf32", pdl));
            else
                MOE_TRY(launch_gemm<EPI_DOWN_ATOMIC>(nmax_dn, mb, a, tiles, s,
                                                     "expert_down_combine_gemm", pdl));
        } else {
            a.out = y_perm;
            a.out_f32 = f32 ? 1 : 0;  // fp32 problems: fp32 weighted rows
            if (f32)
                MOE_TRY(launch_gemm_tf32<EPI_DOWN_STORE>(nmax_dn, mb, a, tiles, s,
                                                         "expert_down_gemm_tf32", pdl));
            else
                MOE_TRY(launch_gemm<EPI_DOWN_STORE>(nmax_dn, mb, a, tiles, s, "expert_down_gemm",
                                                    pdl));
        }
    }
    // 6. token-order output
    if (atomic_combine) {
        if (f32) return run_finalize<float>(out_acc, static_cast<float*>(out), T * H, s, pdl);
        return run_finalize<__nv_bfloat16>(out_acc, static_cast<__nv_bfloat16*>(out), T * H, s,
                                           pdl);
    }
    const int64_t shared_row0 = S ? T * k : -1;
    if (f32)
        return run_gather_sum(static_cast<const float*>(y_perm), pos, T, p->H, p->top_k, T * k,
                              shared_row0, static_cast<float*>(out), status, s, pdl);
    return run_gather_sum(static_cast<const __nv_bfloat16*>(y_perm), pos, T, p->H, p->top_k,
                          T * k, shared_row0, static_cast<__nv_bfloat16*>(out), status, s, pdl);
}

}  // extern "C"

// ------------------------------------------------------------------ routing without allocation
//
// Scratch for moe_route_noalloc: a fixed device array that every GPU which
// loads this library holds until the process exits.  Bytes [0, 256) hold a
// device error word (cleared on each call), the rest the fp32 router logits.
namespace moe {
namespace {
constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;  // 1 MiB
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch on the current device.  In host code
// the array's name only stands in for the symbol; the address is looked up
// once per device (with that device current) and cached.
void* noalloc_scratch_address() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    static std::mutex mu;
    static void* addr[64] = {nullptr};
    std::lock_guard<std::mutex> lk(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return nullptr;
        addr[dev] = p;
    }
    return addr[dev];
}
}  // namespace
}  // namespace moe

extern "C" {

int32_t moe_route_noalloc(const moe_problem* p, const void* x, const void* gate_w,
                          const float* bias, int32_t* topk_idx, float* topk_w, void* stream) {
    MOE_TRY(check_problem(p));
    if (!x || !gate_w || !topk_idx || !topk_w) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(gate_w)) return MOE_ERR_INVALID_ARG;
    const size_t need = 256 + static_cast<size_t>(p->T) * p->E * sizeof(float);
    if (need > kNoAllocScratchBytes) return MOE_ERR_WORKSPACE;
    if (p->T == 0) return MOE_OK;
    uint8_t* base = static_cast<uint8_t*>(noalloc_scratch_address());
    if (!base) return MOE_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t* status = reinterpret_cast<int32_t*>(base);
    float* logits = reinterpret_cast<float*>(base + 256);
    if (cudaMemsetAsync(status, 0, sizeof(int32_t), s) != cudaSuccess) return MOE_ERR_CUDA;
    MOE_TRY(run_logits(p, x, gate_w, logits, status, s));
    return run_topk(p, logits, bias, topk_idx, topk_w, s);
}

int32_t moe_router_stats(const moe_problem* p, const void* x, const void* gate_w,
                         const float* bias, float* P_out, float* f_out, float* aux_out,
                         float* ema_counts, float* ema_total, float momentum, void* ws,
                         size_t ws_bytes, void* stream) {
    MOE_TRY(check_problem(p));
    if (!x || !gate_w || !P_out || !f_out || !aux_out || !ws) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(gate_w) || !aligned16(ws)) return MOE_ERR_INVALID_ARG;
    if (!(momentum >= 0.0f && momentum <= 1.0f)) return MOE_ERR_INVALID_ARG;
    if (p->T == 0) return MOE_ERR_INVALID_ARG;  // a mean over no tokens is undefined
    const Layout L = layout_for(p, MOE_CALL_ROUTER_STATS);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t* status = at<int32_t>(ws, L.status);
    float* logits = at<float>(ws, L.logits);
    int32_t* idx = at<int32_t>(ws, L.idx);
    int32_t* counts = at<int32_t>(ws, L.counts);
    float* partial = at<float>(ws, L.partial);
    MOE_TRY(run_route(p, x, gate_w, bias, logits, at<int32_t>(ws, L.rcount), idx,
                      at<float>(ws, L.w), true, status, s));
    if (cudaMemsetAsync(counts, 0, p->E * sizeof(int32_t), s) != cudaSuccess) return MOE_ERR_CUDA;
    const int nblocks = static_cast<int>((p->T + kStatsTokensPerBlock - 1) / kStatsTokensPerBlock);
    MOE_LAUNCH("router_prob_partial", s,
               router_prob_partial_kernel<<<nblocks, 256, 0, s>>>(logits, bias, idx, p->T, p->E,
                                                                  p->top_k, partial, counts));
    MOE_LAUNCH("router_stats_final", s,
               router_stats_final_kernel<<<1, kMaxExperts, 0, s>>>(
                   partial, nblocks, counts, p->T, p->E, p->top_k, momentum, P_out, f_out,
                   aux_out, ema_counts, ema_total));
    return MOE_OK;
}

int32_t moe_quantize_weights_fp8(const moe_problem* p, int32_t n_experts, const void* w,
                                 uint8_t* q, float* scale_gu, float* scale_d, void* stream) {
    MOE_TRY(check_problem(p));
    if (!w || !q || !scale_gu || !scale_d) return MOE_ERR_INVALID_ARG;
    // the row encoder reads 16-byte vectors of w and writes 8-byte groups of q
    if (!aligned16(w) || !aligned16(q)) return MOE_ERR_INVALID_ARG;
    if (n_experts < 1) return MOE_ERR_INVALID_ARG;
    if (p->H % 128 != 0 || p->I % 128 != 0) return MOE_ERR_UNSUPPORTED;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t I = p->I, H = p->H, n = n_experts;
    // gate and up rows: groups of 2*I rows out of every 3*I
    const int64_t rows = n * 2 * I;
    const unsigned rblocks = static_cast<unsigned>((rows + 7) / 8);
    // down columns: one thread per (expert, column)
    const unsigned cblocks = static_cast<unsigned>((n * H + 255) / 256);
    if (p->dtype == MOE_BF16) {
        const __nv_bfloat16* wb = static_cast<const __nv_bfloat16*>(w);
        MOE_LAUNCH("quantize_weight_rows", s,
                   quantize_rows_e4m3_kernel<__nv_bfloat16><<<rblocks, 256, 0, s>>>(
                       wb, rows, static_cast<int>(H), 2 * I, 3 * I, q, scale_gu));
        MOE_LAUNCH("quantize_weight_cols", s,
                   quantize_cols_e4m3_kernel<__nv_bfloat16><<<cblocks, 256, 0, s>>>(
                       wb + 2 * I * H, 3 * I * H, 3 * I * H, static_cast<int>(n),
                       static_cast<int>(I), static_cast<int>(H), q + 2 * I * H, scale_d));
    } else {
        const float* wf = static_cast<const float*>(w);
        MOE_LAUNCH("quantize_weight_rows", s,
                   quantize_rows_e4m3_kernel<float><<<rblocks, 256, 0, s>>>(
                       wf, rows, static_cast<int>(H), 2 * I, 3 * I, q, scale_gu));
        MOE_LAUNCH("quantize_weight_cols", s,
                   quantize_cols_e4m3_kernel<float><<<cblocks, 256, 0, s>>>(
                       wf + 2 * I * H, 3 * I * H, 3 * I * H, static_cast<int>(n),
                       static_cast<int>(I), static_cast<int>(H), q + 2 * I * H, scale_d));
    }
    return MOE_OK;
}

int32_t moe_forward_fp8(const moe_problem* p, const void* x, const void* gate_w,
                        const float* bias, const uint8_t* expert_q, const float* expert_s_gu,
                        const float* expert_s_d, const uint8_t* shared_q,
                        const float* shared_s_gu, const float* shared_s_d, void* out,
                        int32_t* idx_out, float* w_out, void* ws, size_t ws_bytes,
                        void* stream) {
    MOE_TRY(check_problem(p));
    if (p->dtype != MOE_BF16) return MOE_ERR_UNSUPPORTED;
    if (p->H % 128 != 0 || p->I % 128 != 0) return MOE_ERR_UNSUPPORTED;
    if (!(p->clip_limit > 0.0f && std::isfinite(p->clip_limit))) return MOE_ERR_UNSUPPORTED;
    if (!x || !gate_w || !expert_q || !expert_s_gu || !expert_s_d || !out || !ws)
        return MOE_ERR_INVALID_ARG;
    if (p->num_shared && (!shared_q || !shared_s_gu || !shared_s_d)) return MOE_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(gate_w) || !aligned16(expert_q) || !aligned16(out) ||
        !aligned16(ws) || (shared_q && !aligned16(shared_q)))
        return MOE_ERR_INVALID_ARG;
    const Layout L = layout_for(p, MOE_CALL_FORWARD_FP8);
    if (ws_bytes < L.total) return MOE_ERR_WORKSPACE;
    if (p->T == 0) return MOE_OK;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t* status = at<int32_t>(ws, L.status);
    const int64_t T = p->T, H = p->H, E = p->E, I = p->I, k = p->top_k, S = p->num_shared;
    int32_t* idx = idx_out ? idx_out : at<int32_t>(ws, L.idx);
    float* w = w_out ? w_out : at<float>(ws, L.w);

    // 1. route (bf16 gate GEMM, unquantized)
    MOE_TRY(run_route(p, x, gate_w, bias, at<float>(ws, L.logits), at<int32_t>(ws, L.rcount), idx,
                      w, false, status, s));
    // 2. dispatch
    const int nmax = pick_nmax(static_cast<double>(T * k) / E);
    const int nmax_dn = pick_down_nmax(nmax);
    int32_t* sg = at<int32_t>(ws, L.sched_gu);
    int32_t* sd = at<int32_t>(ws, L.sched_dn);
    int32_t* pos = at<int32_t>(ws, L.pos);
    int32_t* src = at<int32_t>(ws, L.src);
    float* row_w = at<float>(ws, L.row_w);
    MOE_TRY(run_dispatch(p, idx, w, at<int32_t>(ws, L.hist), at<int32_t>(ws, L.base),
                         at<int32_t>(ws, L.counts), at<int32_t>(ws, L.offsets), sg, nmax, sd,
                         nmax_dn, pos, src, row_w, status, s));
    // 3. token rows to E4M3 with a power-of-two scale per token, then permuted
    uint8_t* x_q = at<uint8_t>(ws, L.x_q);
    float* s_x = at<float>(ws, L.s_x);
    MOE_LAUNCH("quantize_tokens", s,
               quantize_rows_e4m3_kernel<__nv_bfloat16><<<static_cast<unsigned>((T + 7) / 8), 256,
                                                          0, s>>>(
                   static_cast<const __nv_bfloat16*>(x), T, static_cast<int>(H), T, T, x_q, s_x));
    uint8_t* x_perm = at<uint8_t>(ws, L.x_perm);
    const bool pdl = pdl_enabled();
    // the gate/up GEMM's gather warps fetch the code rows straight from x_q
    // (as for bf16 rows: tiles of up to 160 rows, MOE_FUSED_GATHER overrides)
    const bool gather_in_gemm = fused_gather(nmax);
    if (!gather_in_gemm)
        MOE_TRY((run_gather<uint8_t, uint8_t>(x_q, T, p->H, p->top_k, pos, T * k, x_perm, nullptr,
                                              nullptr, s, pdl)));
    // 4. gate/up on E4M3 codes; the epilogue applies token x channel scales,
    //    clamps, and writes h as E4M3 with the fixed power-of-two scale
    const double L_clip = p->clip_limit;
    const double hmax = L_clip / (1.0 + std::exp(-L_clip)) * L_clip;
    const float h_scale = static_cast<float>(std::ldexp(1.0, static_cast<int>(
                                                                 std::ceil(std::log2(hmax / 448.0)))));
    uint8_t* h = at<uint8_t>(ws, L.h_perm);
    const int64_t h_rows = T * (k + S);
    const int nseg = static_cast<int>(E + S);
    {
        GemmArgs a = base_args(status);
        if (!make_tmap_gateup(&a.tmA0, expert_q, E * 3, I, H, kU8)) return MOE_ERR_CUDA;
        if (!make_tmap_rows(a.tmB0, x_perm, T * k, H, kU8)) return MOE_ERR_CUDA;
        if (S) {
            if (!make_tmap_gateup(&a.tmA1, shared_q, 3, I, H, kU8)) return MOE_ERR_CUDA;
            if (!make_tmap_rows(a.tmB1, x_q, T, H, kU8)) return MOE_ERR_CUDA;
        } else {
            a.tmA1 = a.tmA0;
            for (int j = 0; j < kNumBoxSizes; ++j) a.tmB1[j] = a.tmB0[j];
        }
        a.sched = sg;
        a.nseg = nseg;
        a.special_seg = S ? static_cast<int32_t>(E) : -1;
        a.K = static_cast<int32_t>(H);
        a.M_total = static_cast<int32_t>(I);
        a.a_seg_stride = 3;
        a.a_off0 = 0;
        a.out = h;
        a.out_ld = static_cast<int32_t>(I);
        a.clip = effective_clip(p);
        a.row_token = src;
        a.routed_rows = static_cast<int32_t>(T * k);
        a.token_scale = s_x;
        a.scale_w = expert_s_gu;
        a.scale_w_special = shared_s_gu;
        a.h_scale = h_scale;
        a.h_scale_inv = 1.0f / h_scale;
        if (gather_in_gemm) {
            a.gather_tok = src;
            a.gather_src = x_q;
            a.n_tokens = static_cast<int32_t>(T);
        }
        expert_gemm_launch_args(a, true);
        MOE_TRY(launch_gemm_fp8<EPI_SWIGLU>(nmax, 2, a, max_tiles(h_rows, nseg, nmax, I), s,
                                            "expert_gate_up_gemm_fp8", pdl));
    }
    // 5. down on E4M3 codes; epilogue: h scale x column scale x routing weight
    __nv_bfloat16* y_perm = at<__nv_bfloat16>(ws, L.y_perm);
    {
        GemmArgs a = base_args(status);
        const int mb = pick_down_mb(nmax_dn);
        if (!make_tmap_down(&a.tmA0, expert_q, E * 3 * I, H, mb, kU8)) return MOE_ERR_CUDA;
        if (!make_tmap_rows(a.tmB0, h, h_rows, I, kU8)) return MOE_ERR_CUDA;
        if (S) {
            if (!make_tmap_down(&a.tmA1, shared_q, 3 * I, H, mb, kU8)) return MOE_ERR_CUDA;
        } else {
            a.tmA1 = a.tmA0;
        }
        for (int j = 0; j < kNumBoxSizes; ++j) a.tmB1[j] = a.tmB0[j];
        a.sched = sd;
        a.nseg = nseg;
        a.special_seg = S ? static_cast<int32_t>(E) : -1;
        a.K = static_cast<int32_t>(I);
        a.M_total = static_cast<int32_t>(H);
        a.a_seg_stride = static_cast<int32_t>(3 * I);
        a.a_off0 = static_cast<int32_t>(2 * I);
        a.out = y_perm;
        a.out_ld = static_cast<int32_t>(H);
        a.n_tokens = static_cast<int32_t>(T);
        a.row_token = src;
        a.row_weight = row_w;
        a.routed_rows = static_cast<int32_t>(T * k);
        a.scale_w = expert_s_d;
        a.scale_w_special = shared_s_d;
        a.h_scale = h_scale;
        a.h_scale_inv = 1.0f / h_scale;
        expert_gemm_launch_args(a, false);
        MOE_TRY(launch_gemm_fp8<EPI_DOWN_STORE>(nmax_dn, mb, a,
                                                max_tiles(h_rows, nseg, nmax_dn, H, 128 * mb), s,
                                                "expert_down_gemm_fp8", pdl));
    }
    // 6. fixed-order combine into token order
    return run_gather_sum(static_cast<const __nv_bfloat16*>(y_perm), pos, T, p->H, p->top_k,
                          T * k, S ? T * k : -1, static_cast<__nv_bfloat16*>(out), status, s,
                          pdl);
}

int32_t moe_read_device_status(const void* ws, int32_t* status_out, void* stream) {
    if (!ws || !status_out) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(status_out, ws, sizeof(int32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
}

int32_t moe_clear_device_status(void* ws, void* stream) {
    if (!ws) return MOE_ERR_INVALID_ARG;
    if (cudaMemsetAsync(ws, 0, sizeof(int32_t), static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}

int32_t moe_check_wait_timeout(void* ws, size_t ws_bytes, int32_t* waits_timed_out,
                               void* stream) {
    if (!ws || !waits_timed_out || ws_bytes < 256 || !aligned16(ws)) return MOE_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint8_t* base = static_cast<uint8_t*>(ws);
    int32_t* status = reinterpret_cast<int32_t*>(base);
    int32_t* counter = reinterpret_cast<int32_t*>(base + 64);
    int32_t* result = reinterpret_cast<int32_t*>(base + 128);
    if (cudaMemsetAsync(base + 64, 0, 128, s) != cudaSuccess) return MOE_ERR_CUDA;
    // about 0.1 s per wait at the B200's clocks
    const uint64_t limit = 200000000ull;
    MOE_LAUNCH("wait_selftest", s,
               wait_selftest_kernel<<<1, 32, 0, s>>>(counter, limit, status, result));
    if (cudaMemcpyAsync(waits_timed_out, result, sizeof(int32_t), cudaMemcpyDeviceToHost, s) !=
        cudaSuccess)
        return MOE_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
}

int64_t moe_launch_count(void) { return g_launches.load(); }

int32_t moe_profile_start(int32_t max_launches) {
    if (max_launches <= 0) return MOE_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(g_prof.mu);
    if (g_prof.on) return MOE_ERR_INVALID_ARG;
    g_prof.pool.assign(2 * static_cast<size_t>(max_launches), nullptr);
    for (auto& e : g_prof.pool) {
        if (cudaEventCreate(&e) != cudaSuccess) return MOE_ERR_CUDA;
    }
    g_prof.recs.clear();
    g_prof.cap = static_cast<size_t>(max_launches);
    g_prof.on = true;
    return MOE_OK;
}

int32_t moe_profile_stop(moe_kernel_time* entries, int32_t max_entries, int32_t* n_entries) {
    std::lock_guard<std::mutex> lk(g_prof.mu);
    if (!g_prof.on) return MOE_ERR_INVALID_ARG;
    g_prof.on = false;
    int32_t rc = MOE_OK;
    int32_t n = 0;
    for (const ProfRecord& r : g_prof.recs) {
        if (cudaEventSynchronize(r.stop) != cudaSuccess) {
            rc = MOE_ERR_CUDA;
            break;
        }
        float ms = 0.0f;
        if (cudaEventElapsedTime(&ms, r.start, r.stop) != cudaSuccess) {
            rc = MOE_ERR_CUDA;
            break;
        }
        int32_t i = 0;
        while (i < n && std::strcmp(entries[i].name, r.name) != 0) ++i;
        if (i == n) {
            if (n >= max_entries) continue;
            entries[n].name = r.name;
            entries[n].launches = 0;
            entries[n].total_ms = 0.0;
            ++n;
        }
        entries[i].launches += 1;
        entries[i].total_ms += ms;
    }
    for (auto& e : g_prof.pool)
        if (e) cudaEventDestroy(e);
    g_prof.pool.clear();
    g_prof.recs.clear();
    if (n_entries) *n_entries = n;
    return rc;
}

}  // extern "C"
