// lbq.cu -- the C ABI (include/lbq.h): argument validation, tensor-map setup,
// tile and split selection, and kernel launches.  One translation unit holds
// every kernel so that the device status word is a single object.
#include <cmath>
#include <cstring>
#include <mutex>
#include <unordered_set>
#include <vector>

#include "dqgemm.cuh"
#include "dqgemm_bwd.cuh"
#include "dqgemv.cuh"
#include "lora.cuh"
#include "merge.cuh"
#include "quantize.cuh"
#include "select.cuh"
#include "selftest.cuh"

using namespace lbq;

namespace {

// ---------------------------------------------------------------------------
// small host helpers
// ---------------------------------------------------------------------------
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }


lbq_status last_launch() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? LBQ_OK : LBQ_ECUDA;
}

int sm_count() {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    return sms > 0 ? sms : 148;
}

// cuTensorMapEncodeTiled, fetched from the driver through the runtime so that
// the library needs no link-time dependency on libcuda.
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 2-D row-major tensor [rows, cols] of `esize`-byte elements, box [brows, bcols].
bool make_map_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dt, int esize, uint64_t rows,
                 uint64_t cols, uint32_t brows, uint32_t bcols, CUtensorMapSwizzle sw) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * static_cast<uint64_t>(esize)};
    cuuint32_t box[2] = {bcols, brows};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Activation view for the forward kernel: bf16 [rows, cols] seen as 3-D
// (64 elements, rows, cols / 64 blocks), box (64, brows, bblocks): one box
// brings `bblocks` consecutive k-blocks of `brows` rows, each k-block landing
// as its own [brows x 128 B] tile (128-byte swizzle).
bool make_map_x3d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t brows,
                  uint32_t bblocks) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {64, rows, cols / 64};
    cuuint64_t strides[2] = {cols * 2, 128};
    cuuint32_t box[3] = {64, brows, bblocks};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---------------------------------------------------------------------------
// weight descriptor checks
// ---------------------------------------------------------------------------
lbq_status check_qweight(const lbq_qweight* q, bool need_data) {
    if (!q) return LBQ_EINVAL;
    if (q->n < 1 || q->k < 64 || q->k % 64 != 0) return LBQ_EINVAL;
    if (q->scheme == LBQ_MINMAX_ASYM) {
        if (!((q->bits == 4 && q->group == 128) || (q->bits == 2 && q->group == 64))) return LBQ_EUNSUPPORTED;
        if (q->k % q->group != 0) return LBQ_EINVAL;
        if (need_data && (!q->packed || !q->scale || !q->zero)) return LBQ_EINVAL;
        if (need_data && (!aligned16(q->packed) || !aligned16(q->scale) || !aligned16(q->zero))) return LBQ_EALIGN;
    } else if (q->scheme == LBQ_CODEBOOK4) {
        if (q->bits != 4 || q->group != 64) return LBQ_EUNSUPPORTED;
        if (need_data && (!q->packed || !q->absmax || !q->codebook)) return LBQ_EINVAL;
        if (need_data && (!aligned16(q->packed) || !aligned16(q->absmax) || !aligned16(q->codebook)))
            return LBQ_EALIGN;
        if (q->double_quant) {
            if (need_data && (!q->absmax_q8 || !q->absmax_s2 || !q->absmax_offset)) return LBQ_EINVAL;
            if (need_data && (!aligned16(q->absmax_q8) || !aligned16(q->absmax_s2) || !aligned16(q->absmax_offset)))
                return LBQ_EALIGN;
        }
    } else {
        return LBQ_EUNSUPPORTED;
    }
    return LBQ_OK;
}

int kind_of(const lbq_qweight* q) {
    if (q->scheme == LBQ_CODEBOOK4) return kCode4;
    return q->bits == 4 ? kInt4 : kInt2;
}

// ---------------------------------------------------------------------------
// forward GEMM planning
// ---------------------------------------------------------------------------
constexpr int kCodebookQuantizeMaxCtas = 4096;

int token_tile(int m) { return m <= 16 ? 16 : m <= 32 ? 32 : m <= 64 ? 64 : m <= 128 ? 128 : 256; }

// Split-K workspace layout, the same for every plan: a fixed header of
// per-tile arrival counters at offset 0, then the fp32 partial sums.  The
// CTA that finishes a tile sets its counter back to zero, so the header stays
// zero between calls whatever shapes share the workspace (partials never land
// on it).
constexpr size_t kCounterHeader = 64 * 1024;
constexpr int kMaxSplitTiles = static_cast<int>(kCounterHeader / sizeof(uint32_t));

inline uint32_t* ws_counters(void* ws) { return static_cast<uint32_t*>(ws); }
inline float* ws_partials(void* ws) { return reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + kCounterHeader); }

// Streams on which the last library call was a quantization: the forward
// that follows on such a stream reads the weight only after that kernel has
// finished.  Any other forward may stream the packed weight while the kernel
// before it on the stream is still running.
std::mutex g_wq_mu;
std::unordered_set<cudaStream_t> g_weights_written;

void note_weights_written(cudaStream_t st) {
    std::lock_guard<std::mutex> lock(g_wq_mu);
    g_weights_written.insert(st);
}

bool weights_stable(cudaStream_t st) {
    std::lock_guard<std::mutex> lock(g_wq_mu);
    return g_weights_written.erase(st) == 0;
}

#include "dqgemv_host.cuh"

// Plan of a tensor-core GEMM (forward: 128-row output tiles, reduction over
// k/64 blocks; backward: 128-feature tiles, reduction over n/64 channel
// blocks), m > 16 or the backward at any m.  Tiles are numbered output tile
// fastest, then token tile.  When the tiles alone cannot fill the CTA slots, every tile's
// reduction is split so that all CTAs fit in one wave (required).  When they
// fill several waves and the last holds a quarter to a half of the slots,
// the full waves run unsplit and the tiles of the last wave are split over
// the idle slots in a second launch, if their partial sums fit `ws_budget`
// bytes of workspace (optional: 512 tiles on 148 slots take 3.5 waves
// instead of 4; a last wave of a few tiles split many ways measured slower,
// as the fixed cost of each CTA and the partial sums outweigh the gain).
// Splits start on a multiple of `align` blocks (the forward's weight chunk);
// the partial sums are [tile - first split tile][split][NT tokens][128] fp32.
struct TilePlan {
    int nt = 0, tiles = 0, rtiles = 0;
    int nsplit = 1, per_split = 0;       // splits of every tile
    int tail0 = 0, tail_split = 1, tail_per = 0;   // tiles tail0 .. tiles - 1, split tail_split ways
    size_t partial_bytes = 0;
    bool split() const { return nsplit > 1 || tail_split > 1; }
    size_t workspace() const { return split() ? kCounterHeader + partial_bytes : 0; }
};

TilePlan plan_tiles(int m, int64_t out_rows, int64_t red, int align, int sms, size_t ws_budget) {
    TilePlan pl;
    pl.nt = std::min(token_tile(m), 256);
    pl.rtiles = static_cast<int>(cdiv(out_rows, 128));
    pl.tiles = static_cast<int>(pl.rtiles * cdiv(m, pl.nt));
    pl.per_split = static_cast<int>(red);
    const int slots = (pl.nt >= 256 ? 1 : 2) * sms;
    auto per_for = [&](int64_t ns) { return static_cast<int>(cdiv(cdiv(red, ns), align) * align); };
    auto bytes_for = [&](int64_t tiles, int ns) {
        return round_up(static_cast<size_t>(tiles) * ns * pl.nt * 128 * sizeof(float), 256);
    };
    if (pl.tiles < slots) {
        pl.per_split = per_for(std::min<int64_t>(red, std::max(1, slots / pl.tiles)));
        pl.nsplit = static_cast<int>(cdiv(red, pl.per_split));
        if (pl.nsplit > 1) pl.partial_bytes = bytes_for(pl.tiles, pl.nsplit);
        return pl;
    }
    const int full = pl.tiles / slots * slots, tail = pl.tiles - full;
    if (2 * tail > slots || 4 * tail < slots || pl.tiles > kMaxSplitTiles) return pl;
    const int per = per_for(slots / tail);
    const int ns = static_cast<int>(cdiv(red, per));
    if (ns < 2 || kCounterHeader + bytes_for(tail, ns) > ws_budget) return pl;
    pl.tail0 = full;
    pl.tail_split = ns;
    pl.tail_per = per;
    pl.partial_bytes = bytes_for(tail, ns);
    return pl;
}

TilePlan plan_fwd(int m, const lbq_qweight* q, int sms, size_t ws_budget = ~size_t(0)) {
    return plan_tiles(m, q->n, q->k / 64, q->bits == 2 ? 8 : 4, sms, ws_budget);
}

TilePlan plan_bwd(int m, const lbq_qweight* q, int sms, size_t ws_budget = ~size_t(0)) {
    return plan_tiles(m, q->k, cdiv(q->n, 64), 1, sms, ws_budget);
}

// Workspace of one forward call (either path): with ws_budget = 0 the part
// that a call requires, unbounded the size that also lets it split the tiles
// of its last wave (what the size queries report).
size_t fwd_workspace(int m, const lbq_qweight* q, int sms, size_t ws_budget = ~size_t(0)) {
    if (m <= kGemvMaxM) return gemv_jobs_workspace(m, &q, 1, sms);
    return plan_fwd(m, q, sms, ws_budget).workspace();
}

template <int NT, int KIND>
lbq_status launch_fwd_nt(const FwdParams& p, const void* X, int m, int64_t k, const uint8_t* packed, int nrows,
                         int nctas, cudaStream_t st) {
    using C = FwdCfg<NT>;
    using L = FwdSmem<NT, C::kXStages, C::kXBlocks, C::kWStages, C::kAStages>;
    auto kern = dqgemm_fwd_kernel<NT, KIND, C::kXStages, C::kXBlocks, C::kWStages, C::kAStages, C::kMinBlocks,
                                  C::kDqWarps>;
    const size_t smem = L::total(p.rank);
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
        return LBQ_ECUDA;
    CUtensorMap tmX, tmW;
    if (!make_map_x3d(&tmX, X, m, k, NT, C::kXBlocks)) return LBQ_ECUDA;
    if (!make_map_2d(&tmW, packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, nrows, k * (KIND == kInt2 ? 2 : 4) / 8, 128, 128,
                     CU_TENSOR_MAP_SWIZZLE_128B))
        return LBQ_ECUDA;
    (void)m;
    kern<<<static_cast<unsigned>(nctas), fwd_threads(C::kDqWarps), smem, st>>>(tmX, tmW, p);
    return last_launch();
}

template <int KIND>
lbq_status launch_fwd_kind(int nt, const FwdParams& p, const void* X, int m, int64_t k, const uint8_t* packed,
                           int nrows, int nctas, cudaStream_t st) {
    switch (nt) {
        case 16: return launch_fwd_nt<16, KIND>(p, X, m, k, packed, nrows, nctas, st);
        case 32: return launch_fwd_nt<32, KIND>(p, X, m, k, packed, nrows, nctas, st);
        case 64: return launch_fwd_nt<64, KIND>(p, X, m, k, packed, nrows, nctas, st);
        case 128: return launch_fwd_nt<128, KIND>(p, X, m, k, packed, nrows, nctas, st);
        default: return launch_fwd_nt<256, KIND>(p, X, m, k, packed, nrows, nctas, st);
    }
}

// The kernel arguments of one forward GEMM, without a K split.
FwdParams fwd_params(int m, const lbq_qweight* q, const void* B, int rank, float s, const float* T, float* Y,
                     int64_t ldy, const int32_t* perm) {
    FwdParams p{};
    p.m = m;
    p.n = q->n;
    p.k = q->k;
    p.ngroups = q->scheme == LBQ_MINMAX_ASYM ? q->k / q->group : 0;
    p.scale = q->scale;
    p.zero = q->zero;
    p.absmax = q->absmax;
    p.q8 = (q->scheme == LBQ_CODEBOOK4 && q->double_quant) ? q->absmax_q8 : nullptr;
    p.s2 = q->absmax_s2;
    p.offset = q->absmax_offset;
    p.codebook = q->codebook;
    p.rank = rank;
    p.rank_pad = rank > 0 ? (rank + 15) / 16 * 16 : 16;
    p.s = s;
    p.T = T;
    p.B = static_cast<const uint16_t*>(B);
    p.Y = Y;
    p.ldy = ldy;
    p.perm = perm;
    p.kb_per_split = q->k / 64;
    p.nsplit = 1;
    return p;
}

lbq_status run_fwd_gemm(const void* X, int m, const lbq_qweight* q, const void* B, int rank, float s,
                        const float* T, float* Y, int64_t ldy, const int32_t* perm, void* ws, size_t ws_bytes,
                        int sms, cudaStream_t st) {
    if (m <= kGemvMaxM) {
        const GvJob job{X, q, B, rank, s, T, Y, ldy, perm};
        return run_gemv_jobs(m, &job, 1, ws, ws_bytes, sms, st);
    }
    const TilePlan pl = plan_fwd(m, q, sms, ws && aligned16(ws) ? ws_bytes : 0);
    FwdParams p = fwd_params(m, q, B, rank, s, T, Y, ldy, perm);
    p.rtiles = pl.rtiles;
    if (pl.split()) {
        if (!ws) return LBQ_EWORKSPACE;
        if (pl.tiles > kMaxSplitTiles) return LBQ_EUNSUPPORTED;
        p.partial = ws_partials(ws);
        p.counters = ws_counters(ws);
    }
    auto launch = [&](const FwdParams& lp, int nctas) {
        switch (kind_of(q)) {
            case kInt4: return launch_fwd_kind<kInt4>(pl.nt, lp, X, m, q->k, q->packed, q->n, nctas, st);
            case kInt2: return launch_fwd_kind<kInt2>(pl.nt, lp, X, m, q->k, q->packed, q->n, nctas, st);
            default: return launch_fwd_kind<kCode4>(pl.nt, lp, X, m, q->k, q->packed, q->n, nctas, st);
        }
    };
    p.kb_per_split = pl.per_split;
    p.nsplit = pl.nsplit;
    if (pl.tail_split <= 1) return launch(p, pl.tiles * pl.nsplit);
    // the full waves unsplit, then the last wave's tiles split over the slots
    lbq_status r = launch(p, pl.tail0);
    if (r != LBQ_OK) return r;
    FwdParams t = p;
    t.tile0 = pl.tail0;
    t.nsplit = pl.tail_split;
    t.kb_per_split = pl.tail_per;
    return launch(t, (pl.tiles - pl.tail0) * pl.tail_split);
}

// One grouped launch of the forward GEMM over g.count problems.
template <int NT>
lbq_status launch_fwd_group_nt(const FwdGroupParams& g, bool any_rank, cudaStream_t st) {
    using C = FwdCfg<NT>;
    using L = FwdSmem<NT, C::kXStages, C::kXBlocks, C::kWStages, C::kAStages>;
    auto kern = dqgemm_fwd_grouped_kernel<NT, C::kXStages, C::kXBlocks, C::kWStages, C::kAStages, C::kMinBlocks,
                                          C::kDqWarps>;
    const size_t smem = L::total(any_rank ? 1 : 0);
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
        return LBQ_ECUDA;
    kern<<<static_cast<unsigned>(g.cta0[g.count]), fwd_threads(C::kDqWarps), smem, st>>>(g);
    return last_launch();
}

template <int NT>
lbq_status run_fwd_group_nt(int m, const GvJob* jobs, int count, cudaStream_t st) {
    using C = FwdCfg<NT>;
    FwdGroupParams g;                                    // passed by value at launch
    memset(&g, 0, sizeof(g));
    g.count = count;
    bool any_rank = false;
    int cta = 0;
    for (int i = 0; i < count; ++i) {
        const GvJob& j = jobs[i];
        const lbq_qweight* q = j.q;
        if (!make_map_x3d(&g.tmX[i], j.X, m, q->k, NT, C::kXBlocks)) return LBQ_ECUDA;
        if (!make_map_2d(&g.tmW[i], q->packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, q->n,
                         static_cast<int64_t>(q->k) * q->bits / 8, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B))
            return LBQ_ECUDA;
        g.p[i] = fwd_params(m, q, j.B, j.rank, j.s, j.T, j.Y, j.ldy, j.perm);
        g.kind[i] = kind_of(q);
        g.rtiles[i] = static_cast<int>(cdiv(q->n, 128));
        g.cta0[i] = cta;
        cta += g.rtiles[i] * static_cast<int>(cdiv(m, NT));
        any_rank |= j.rank > 0;
    }
    g.cta0[count] = cta;
    return launch_fwd_group_nt<NT>(g, any_rank, st);
}

// Forward GEMMs with one token count m > 16 (several matrices, or the two
// halves of channel-mix weights).  When their output tiles together fill the
// machine's CTA slots they run as grouped launches of up to kFwdMaxGroup
// problems, without K splits; otherwise one launch each, with the split that
// fills the machine.
lbq_status run_fwd_jobs(int m, const GvJob* jobs, int count, void* ws, size_t ws_bytes, int sms, cudaStream_t st) {
    const int nt = std::min(token_tile(m), 256);
    const int slots = (nt >= 256 ? 1 : 2) * sms;
    int64_t tiles = 0;
    for (int i = 0; i < count; ++i) tiles += cdiv(jobs[i].q->n, 128) * cdiv(m, nt);
    lbq_status s = LBQ_OK;
    if (count < 2 || tiles < slots) {
        for (int i = 0; i < count && s == LBQ_OK; ++i) {
            const GvJob& j = jobs[i];
            s = run_fwd_gemm(j.X, m, j.q, j.B, j.rank, j.s, j.T, j.Y, j.ldy, j.perm, ws, ws_bytes, sms, st);
        }
        return s;
    }
    for (int i = 0; i < count && s == LBQ_OK; i += kFwdMaxGroup) {
        const int c = std::min(kFwdMaxGroup, count - i);
        switch (nt) {
            case 32: s = run_fwd_group_nt<32>(m, jobs + i, c, st); break;
            case 64: s = run_fwd_group_nt<64>(m, jobs + i, c, st); break;
            case 128: s = run_fwd_group_nt<128>(m, jobs + i, c, st); break;
            default: s = run_fwd_group_nt<256>(m, jobs + i, c, st); break;
        }
    }
    return s;
}

lbq_status check_lora(int rank, const void* A, const void* B, const void* saved) {
    if (rank < 0 || rank > kLoraMaxRank) return LBQ_EINVAL;
    if (rank == 0) return LBQ_OK;
    if (!A || !B || !saved) return LBQ_EINVAL;
    if (!aligned16(A) || !aligned16(B) || !aligned16(saved)) return LBQ_EALIGN;
    return LBQ_OK;
}

// ---------------------------------------------------------------------------
// backward GEMM
// ---------------------------------------------------------------------------
template <int NT, int KIND>
lbq_status launch_bwd_nt(const BwdParams& p, const void* dY, const uint8_t* packed, int nctas, cudaStream_t st) {
    constexpr int BITS = KIND == kInt2 ? 2 : 4;
    using C = BwdCfg<NT>;
    using L = BwdSmem<NT, BITS, C::kXStages, C::kWStages, C::kAStages>;
    auto kern = dqgemm_bwd_kernel<NT, KIND, C::kXStages, C::kWStages, C::kAStages, C::kMinBlocks, C::kDqWarps>;
    const size_t smem = L::total(p.rank_pad);
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
        return LBQ_ECUDA;
    CUtensorMap tmDY, tmW;
    if (!make_map_2d(&tmDY, dY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, p.m, p.n, NT, 64, CU_TENSOR_MAP_SWIZZLE_128B))
        return LBQ_ECUDA;
    if (!make_map_2d(&tmW, packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, p.n, static_cast<int64_t>(p.k) * BITS / 8, 64,
                     L::kKTB, CU_TENSOR_MAP_SWIZZLE_NONE))
        return LBQ_ECUDA;
    kern<<<static_cast<unsigned>(nctas), fwd_threads(C::kDqWarps), smem, st>>>(tmDY, tmW, p);
    return last_launch();
}

template <int KIND>
lbq_status launch_bwd_kind(int nt, const BwdParams& p, const void* dY, const uint8_t* packed, int nctas,
                           cudaStream_t st) {
    switch (nt) {
        case 16: return launch_bwd_nt<16, KIND>(p, dY, packed, nctas, st);
        case 32: return launch_bwd_nt<32, KIND>(p, dY, packed, nctas, st);
        case 64: return launch_bwd_nt<64, KIND>(p, dY, packed, nctas, st);
        case 128: return launch_bwd_nt<128, KIND>(p, dY, packed, nctas, st);
        default: return launch_bwd_nt<256, KIND>(p, dY, packed, nctas, st);
    }
}

// The kernel arguments of one backward GEMM, without a channel split.
BwdParams bwd_params(int m, const lbq_qweight* q, const void* A, int rank, float s, const float* U, float* dX) {
    BwdParams p{};
    p.m = m;
    p.n = q->n;
    p.k = q->k;
    p.bits = q->bits;
    p.ngroups = q->k / q->group;
    p.group = q->group;
    p.scale = q->scale;
    p.zero = q->zero;
    p.absmax = q->absmax;
    p.q8 = (q->scheme == LBQ_CODEBOOK4 && q->double_quant) ? q->absmax_q8 : nullptr;
    p.s2 = q->absmax_s2;
    p.offset = q->absmax_offset;
    p.codebook = q->codebook;
    p.rank = rank;
    p.rank_pad = rank > 0 ? (rank + 15) / 16 * 16 : 16;
    p.s = s;
    p.U = U;
    p.A = static_cast<const uint16_t*>(A);
    p.dX = dX;
    p.cb_per_split = static_cast<int>(cdiv(q->n, 64));
    p.nsplit = 1;
    return p;
}

// One backward GEMM (the adapter's U already computed), with the channel
// split its plan gives.
lbq_status run_bwd_gemm(const void* dY, int m, const lbq_qweight* q, const void* A, int rank, float s, const float* U,
                        float* dX, void* ws, size_t ws_bytes, int sms, cudaStream_t st) {
    const TilePlan pl = plan_bwd(m, q, sms, ws && aligned16(ws) ? ws_bytes : 0);
    BwdParams p = bwd_params(m, q, A, rank, s, U, dX);
    p.ftiles = pl.rtiles;
    if (pl.split()) {
        if (!ws) return LBQ_EWORKSPACE;
        if (pl.tiles > kMaxSplitTiles) return LBQ_EUNSUPPORTED;
        p.partial = ws_partials(ws);
        p.counters = ws_counters(ws);
    }
    auto launch = [&](const BwdParams& lp, int nctas) {
        switch (kind_of(q)) {
            case kInt4: return launch_bwd_kind<kInt4>(pl.nt, lp, dY, q->packed, nctas, st);
            case kInt2: return launch_bwd_kind<kInt2>(pl.nt, lp, dY, q->packed, nctas, st);
            default: return launch_bwd_kind<kCode4>(pl.nt, lp, dY, q->packed, nctas, st);
        }
    };
    p.cb_per_split = pl.per_split;
    p.nsplit = pl.nsplit;
    if (pl.tail_split <= 1) return launch(p, pl.tiles * pl.nsplit);
    // the full waves unsplit, then the last wave's tiles split over the slots
    lbq_status r = launch(p, pl.tail0);
    if (r != LBQ_OK) return r;
    BwdParams t = p;
    t.tile0 = pl.tail0;
    t.nsplit = pl.tail_split;
    t.cb_per_split = pl.tail_per;
    return launch(t, (pl.tiles - pl.tail0) * pl.tail_split);
}

// One grouped launch of the backward GEMM over `count` problems.
template <int NT>
lbq_status run_bwd_group_nt(int m, const lbq_bwd_problem* probs, int count, cudaStream_t st) {
    using C = BwdCfg<NT>;
    BwdGroupParams g;                                    // passed by value at launch
    memset(&g, 0, sizeof(g));
    g.count = count;
    size_t smem = 0;
    int cta = 0;
    for (int i = 0; i < count; ++i) {
        const lbq_bwd_problem& pr = probs[i];
        const lbq_qweight* q = pr.q;
        const bool int2 = kind_of(q) == kInt2;
        const int ktb = 128 * (int2 ? 2 : 4) / 8;        // packed bytes of a channel row across a feature tile
        if (!make_map_2d(&g.tmDY[i], pr.dY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, m, q->n, NT, 64,
                         CU_TENSOR_MAP_SWIZZLE_128B))
            return LBQ_ECUDA;
        if (!make_map_2d(&g.tmW[i], q->packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, q->n,
                         static_cast<int64_t>(q->k) * (int2 ? 2 : 4) / 8, 64, ktb, CU_TENSOR_MAP_SWIZZLE_NONE))
            return LBQ_ECUDA;
        g.p[i] = bwd_params(m, q, pr.A, pr.rank, pr.s, pr.U_save, pr.dX);
        g.kind[i] = kind_of(q);
        g.ftiles[i] = static_cast<int>(cdiv(q->k, 128));
        g.cta0[i] = cta;
        cta += g.ftiles[i] * static_cast<int>(cdiv(m, NT));
        smem = std::max(smem, int2 ? BwdSmem<NT, 2, C::kXStages, C::kWStages, C::kAStages>::total(g.p[i].rank_pad)
                                   : BwdSmem<NT, 4, C::kXStages, C::kWStages, C::kAStages>::total(g.p[i].rank_pad));
    }
    g.cta0[count] = cta;
    auto kern = dqgemm_bwd_grouped_kernel<NT, C::kXStages, C::kWStages, C::kAStages, C::kMinBlocks, C::kDqWarps>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
        return LBQ_ECUDA;
    kern<<<static_cast<unsigned>(cta), fwd_threads(C::kDqWarps), smem, st>>>(g);
    return last_launch();
}

// Checks of one backward problem (as lbq_linear_bwd's).
lbq_status check_bwd(const void* dY, int m, const lbq_qweight* q, const void* A, const void* B, int rank,
                     const float* dX, const float* U_save) {
    lbq_status st = check_qweight(q, true);
    if (st != LBQ_OK) return st;
    if (m < 1 || !dY || !dX || q->n % 8 != 0) return LBQ_EINVAL;
    if (!aligned16(dY) || !aligned16(dX)) return LBQ_EALIGN;
    return check_lora(rank, A, B, U_save);
}

}  // namespace

// ---------------------------------------------------------------------------
// Fixed scratch of lbq_linear_fwd_noalloc.  Every device that loads this
// library holds one copy until the process exits.  In host code the name
// below is only a stand-in for the symbol; the device address of the current
// device's copy comes from cudaGetSymbolAddress, with that device current, on
// every call.  Both split-K paths of the forward (the decode GEMV and the
// tensor-core GEMM) use it as their workspace.
// ---------------------------------------------------------------------------
static constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
// The device address of the current device's copy of the array, looked up on
// every call (a host-side lookup: no allocation, no synchronization once the
// library's module is loaded on the device), so that a reloaded module after
// a context teardown is never addressed through a stale pointer.
lbq_status noalloc_scratch_address(void** out) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return LBQ_ECUDA;
    *out = p;
    return LBQ_OK;
}
}  // namespace

// ===========================================================================
// C ABI
// ===========================================================================
// T = X A^T (row layout) or U = dY B (col layout), [m, rank] fp32.  Decode
// sizes use one CTA per row; larger batches the tensor-core kernel.
template <bool kCol, int R8>
void launch_lora_rows_r8(const uint16_t* in, int64_t m, int64_t len, const uint16_t* wt, int r, float* out,
                         cudaStream_t st) {
    lora_rows_mma_kernel<kCol, R8><<<static_cast<unsigned>(cdiv(m, 16)), 256, 0, st>>>(in, m, len, wt, r, out);
}

template <bool kCol>
lbq_status launch_lora_rows(const void* in, int64_t m, int64_t len, const void* wt, int r, float* out,
                            cudaStream_t st) {
    const uint16_t* a = static_cast<const uint16_t*>(in);
    const uint16_t* w = static_cast<const uint16_t*>(wt);
    if (m < 32) {
        lora_rowdot_kernel<kCol><<<static_cast<unsigned>(m), 256, 0, st>>>(a, len, w, r, out);
        return last_launch();
    }
    switch ((r + 7) / 8) {
        case 1: launch_lora_rows_r8<kCol, 1>(a, m, len, w, r, out, st); break;
        case 2: launch_lora_rows_r8<kCol, 2>(a, m, len, w, r, out, st); break;
        case 3: launch_lora_rows_r8<kCol, 3>(a, m, len, w, r, out, st); break;
        case 4: launch_lora_rows_r8<kCol, 4>(a, m, len, w, r, out, st); break;
        case 5: launch_lora_rows_r8<kCol, 5>(a, m, len, w, r, out, st); break;
        case 6: launch_lora_rows_r8<kCol, 6>(a, m, len, w, r, out, st); break;
        case 7: launch_lora_rows_r8<kCol, 7>(a, m, len, w, r, out, st); break;
        default: launch_lora_rows_r8<kCol, 8>(a, m, len, w, r, out, st); break;
    }
    return last_launch();
}

template <int R8>
void launch_lora_colgrad_r8(const uint16_t* in, int64_t m, int64_t ncols, const float* coef, int r, float s,
                            float* grad, int64_t ocs, int64_t ots, cudaStream_t st) {
    auto kern = lora_colgrad_mma_kernel<R8>;
    const int smem = ColGradSmem<R8>::kBytes;
    cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(cdiv(ncols, 32)), kLoraSplit, 1);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = kLoraSplit;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaLaunchKernelEx(&cfg, kern, in, m, ncols, coef, r, s, grad, ocs, ots);
}

lbq_status launch_lora_colgrad(const void* in, int64_t m, int64_t ncols, const float* coef, int r, float s,
                               float* grad, int64_t ocs, int64_t ots, cudaStream_t st) {
    const uint16_t* a = static_cast<const uint16_t*>(in);
    if (r % 4 != 0) {
        // coefficient rows are copied in 16-byte pieces: ranks that are not a
        // multiple of 4 take the plain kernel
        lora_colgrad_kernel<<<static_cast<unsigned>(cdiv(ncols, 32)), 256, 0, st>>>(a, m, ncols, coef, r, s, grad,
                                                                                    ocs, ots);
        return last_launch();
    }
    switch ((r + 7) / 8) {
        case 1: launch_lora_colgrad_r8<1>(a, m, ncols, coef, r, s, grad, ocs, ots, st); break;
        case 2: launch_lora_colgrad_r8<2>(a, m, ncols, coef, r, s, grad, ocs, ots, st); break;
        case 3: launch_lora_colgrad_r8<3>(a, m, ncols, coef, r, s, grad, ocs, ots, st); break;
        case 4: launch_lora_colgrad_r8<4>(a, m, ncols, coef, r, s, grad, ocs, ots, st); break;
        case 5: launch_lora_colgrad_r8<5>(a, m, ncols, coef, r, s, grad, ocs, ots, st); break;
        case 6: launch_lora_colgrad_r8<6>(a, m, ncols, coef, r, s, grad, ocs, ots, st); break;
        case 7: launch_lora_colgrad_r8<7>(a, m, ncols, coef, r, s, grad, ocs, ots, st); break;
        default: launch_lora_colgrad_r8<8>(a, m, ncols, coef, r, s, grad, ocs, ots, st); break;
    }
    return last_launch();
}

namespace {

// The workspace of a channel-mix forward (both halves); ws_budget as for
// fwd_workspace.
size_t mix_workspace(int m, const lbq_qweight_mix* q, int sms, size_t ws_budget = ~size_t(0)) {
    if (m <= kGemvMaxM) {
        const lbq_qweight* qs[2] = {&q->hi, &q->lo};
        return gemv_jobs_workspace(m, qs, 2, sms);
    }
    return std::max(plan_fwd(m, &q->hi, sms, ws_budget).workspace(), plan_fwd(m, &q->lo, sms, ws_budget).workspace());
}

// Validation of one channel-mix problem's descriptor, activations and outputs.
lbq_status check_mix(const lbq_qweight_mix* q, int m, const void* X, const float* Y) {
    if (!q || !q->perm) return LBQ_EINVAL;
    lbq_status st;
    if ((st = check_qweight(&q->hi, true)) != LBQ_OK) return st;
    if ((st = check_qweight(&q->lo, true)) != LBQ_OK) return st;
    if (q->hi.scheme != LBQ_MINMAX_ASYM || q->lo.scheme != LBQ_MINMAX_ASYM || q->hi.k != q->lo.k) return LBQ_EINVAL;
    if (m < 1 || !X || !Y) return LBQ_EINVAL;
    if (!aligned16(X) || !aligned16(Y) || !aligned16(q->perm)) return LBQ_EALIGN;
    return LBQ_OK;
}

}  // namespace

extern "C" {

const char* lbq_status_string(lbq_status s) {
    switch (s) {
        case LBQ_OK: return "ok";
        case LBQ_EINVAL: return "invalid argument";
        case LBQ_EALIGN: return "device pointer not 16-byte aligned";
        case LBQ_EUNSUPPORTED: return "unsupported configuration";
        case LBQ_ECUDA: return "CUDA error";
        case LBQ_ETIMEOUT: return "device-side wait timed out";
        case LBQ_EWORKSPACE: return "workspace missing or too small";
    }
    return "unknown status";
}

size_t lbq_quantize_workspace_size(const lbq_qweight* q) {
    if (q && q->scheme == LBQ_CODEBOOK4 && q->double_quant) return kCodebookQuantizeMaxCtas * sizeof(double);
    return 0;
}

lbq_status lbq_quantize(const void* W_bf16, lbq_qweight* q, void* workspace, size_t workspace_bytes,
                        lbq_stream_t stream) {
    lbq_status st = check_qweight(q, true);
    if (st != LBQ_OK) return st;
    if (!W_bf16) return LBQ_EINVAL;
    if (!aligned16(W_bf16)) return LBQ_EALIGN;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    note_weights_written(s);
    const int64_t nchunks = static_cast<int64_t>(q->n) * q->k / 8;
    const int sms = sm_count();
    if (q->scheme == LBQ_MINMAX_ASYM) {
        const int grid = static_cast<int>(std::min<int64_t>(cdiv(nchunks, 256), 16LL * sms));
        if (q->bits == 4)
            minmax_quantize_kernel<4><<<grid, 256, 0, s>>>(static_cast<const uint4*>(W_bf16), nchunks, q->packed,
                                                            q->scale, q->zero);
        else
            minmax_quantize_kernel<2><<<grid, 256, 0, s>>>(static_cast<const uint4*>(W_bf16), nchunks, q->packed,
                                                            q->scale, q->zero);
        return last_launch();
    }
    const int grid = static_cast<int>(std::min<int64_t>(cdiv(nchunks, 256), std::min(16 * sms, kCodebookQuantizeMaxCtas)));
    double* sums = nullptr;
    if (q->double_quant) {
        if (!workspace || workspace_bytes < lbq_quantize_workspace_size(q)) return LBQ_EWORKSPACE;
        if (!aligned16(workspace)) return LBQ_EALIGN;
        sums = static_cast<double*>(workspace);
    }
    codebook_quantize_kernel<<<grid, 256, 0, s>>>(static_cast<const uint4*>(W_bf16), nchunks, q->codebook, q->packed,
                                                  q->absmax, sums);
    if ((st = last_launch()) != LBQ_OK) return st;
    if (q->double_quant) {
        const int64_t nb = static_cast<int64_t>(q->n) * q->k / 64;
        absmax_offset_kernel<<<1, 256, 0, s>>>(sums, grid, nb, q->absmax_offset);
        if ((st = last_launch()) != LBQ_OK) return st;
        double_quant_kernel<<<static_cast<unsigned>(cdiv(nb, 256)), 256, 0, s>>>(q->absmax, nb, q->absmax_offset,
                                                                                q->absmax_q8, q->absmax_s2);
        return last_launch();
    }
    return LBQ_OK;
}

lbq_status lbq_dequantize(const lbq_qweight* q, float* W_f32, lbq_stream_t stream) {
    lbq_status st = check_qweight(q, true);
    if (st != LBQ_OK) return st;
    if (!W_f32) return LBQ_EINVAL;
    if (!aligned16(W_f32)) return LBQ_EALIGN;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int64_t nchunks = static_cast<int64_t>(q->n) * q->k / 8;
    const int grid = static_cast<int>(std::min<int64_t>(cdiv(nchunks, 256), 16LL * sm_count()));
    float4* out = reinterpret_cast<float4*>(W_f32);
    if (q->scheme == LBQ_MINMAX_ASYM) {
        if (q->bits == 4)
            minmax_dequantize_kernel<4><<<grid, 256, 0, s>>>(q->packed, q->scale, q->zero, nchunks, out);
        else
            minmax_dequantize_kernel<2><<<grid, 256, 0, s>>>(q->packed, q->scale, q->zero, nchunks, out);
    } else {
        codebook_dequantize_kernel<<<grid, 256, 0, s>>>(q->packed, q->absmax, q->double_quant ? q->absmax_q8 : nullptr,
                                                        q->absmax_s2, q->absmax_offset, q->codebook, nchunks, out);
    }
    return last_launch();
}

// Merge grid: one CTA per 64-row x 128-column tile (n / 64 <= 65535 rows of tiles).
dim3 merge_grid(int n, int k) {
    return dim3(static_cast<unsigned>(cdiv(k, kMergeCols)), static_cast<unsigned>(cdiv(n, kMergeRows)));
}

lbq_status lbq_merge_lora(const lbq_qweight* q, const void* A, const void* B, int rank, float s, void* W_out,
                          lbq_stream_t stream) {
    lbq_status st = check_qweight(q, true);
    if (st != LBQ_OK) return st;
    if (!W_out || rank < 0 || rank > kLoraMaxRank || (rank > 0 && (!A || !B))) return LBQ_EINVAL;
    if (!aligned16(W_out) || (rank > 0 && (!aligned16(A) || !aligned16(B)))) return LBQ_EALIGN;
    MergeParams p{};
    p.n = q->n;
    p.k = q->k;
    p.ngroups = q->scheme == LBQ_MINMAX_ASYM ? q->k / q->group : 0;
    p.packed = q->packed;
    p.scale = q->scale;
    p.zero = q->zero;
    p.absmax = q->absmax;
    p.q8 = (q->scheme == LBQ_CODEBOOK4 && q->double_quant) ? q->absmax_q8 : nullptr;
    p.s2 = q->absmax_s2;
    p.offset = q->absmax_offset;
    p.codebook = q->codebook;
    p.A = static_cast<const uint16_t*>(A);
    p.B = static_cast<const uint16_t*>(B);
    p.rank = rank;
    p.s = s;
    p.out = static_cast<uint16_t*>(W_out);
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    const dim3 grid = merge_grid(q->n, q->k);
    if (grid.y > 65535u) return LBQ_EUNSUPPORTED;
    if (q->scheme == LBQ_MINMAX_ASYM) {
        if (q->bits == 4)
            lora_merge_kernel<kMergeInt4><<<grid, kMergeThreads, 0, cs>>>(p);
        else
            lora_merge_kernel<kMergeInt2><<<grid, kMergeThreads, 0, cs>>>(p);
    } else {
        lora_merge_kernel<kMergeCode4><<<grid, kMergeThreads, 0, cs>>>(p);
    }
    return last_launch();
}

lbq_status lbq_unmerge_lora(const void* W, int n, int k, const void* A, const void* B, int rank, float s, void* W_out,
                            lbq_stream_t stream) {
    if (!W || !W_out || n < 1 || k < 8 || k % 8 != 0) return LBQ_EINVAL;
    if (rank < 0 || rank > kLoraMaxRank || (rank > 0 && (!A || !B))) return LBQ_EINVAL;
    if (!aligned16(W) || !aligned16(W_out) || (rank > 0 && (!aligned16(A) || !aligned16(B)))) return LBQ_EALIGN;
    MergeParams p{};
    p.n = n;
    p.k = k;
    p.W = static_cast<const uint16_t*>(W);
    p.A = static_cast<const uint16_t*>(A);
    p.B = static_cast<const uint16_t*>(B);
    p.rank = rank;
    p.s = s;
    p.out = static_cast<uint16_t*>(W_out);
    const dim3 grid = merge_grid(n, k);
    if (grid.y > 65535u) return LBQ_EUNSUPPORTED;
    lora_merge_kernel<kMergeBf16><<<grid, kMergeThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(p);
    return last_launch();
}

size_t lbq_linear_fwd_workspace_size(int m, const lbq_qweight* q, int rank) {
    (void)rank;
    if (m < 1 || check_qweight(q, false) != LBQ_OK) return 0;
    return fwd_workspace(m, q, sm_count());
}

lbq_status lbq_gemv_plan(int m, const lbq_qweight* const* qs, int count, int sms, int64_t* plan,
                         int64_t* per_problem) {
    if (m < 1 || m > kGemvMaxM || !qs || !plan || count < 1 || count > kGvMaxProblems) return LBQ_EINVAL;
    for (int i = 0; i < count; ++i)
        if (check_qweight(qs[i], false) != LBQ_OK) return LBQ_EINVAL;
    if (sms <= 0) sms = sm_count();
    GvPlan pl;
    const lbq_status st = gv_plan(m, qs, count, sms, &pl);
    if (st != LBQ_OK) return st;
    plan[0] = pl.ctas;
    plan[1] = pl.ws;
    plan[2] = pl.stage_bytes;
    plan[3] = static_cast<int64_t>(pl.smem);
    plan[4] = static_cast<int64_t>(pl.workspace);
    plan[5] = sms;
    plan[6] = pl.xbox_max;
    plan[7] = pl.cstride;
    if (per_problem) {
        for (int i = 0; i < count; ++i) {
            per_problem[4 * i + 0] = pl.share[i];
            per_problem[4 * i + 1] = pl.pctas[i];
            per_problem[4 * i + 2] = pl.cta0[i];
            per_problem[4 * i + 3] = pl.tiles[i];
        }
    }
    return LBQ_OK;
}

lbq_status lbq_linear_fwd(const void* X, int m, const lbq_qweight* q, const void* A, const void* B, int rank,
                          float s, float* Y, float* T_save, void* workspace, size_t workspace_bytes,
                          lbq_stream_t stream) {
    lbq_status st = check_qweight(q, true);
    if (st != LBQ_OK) return st;
    if (m < 1 || !X || !Y) return LBQ_EINVAL;
    if (!aligned16(X) || !aligned16(Y)) return LBQ_EALIGN;
    if ((st = check_lora(rank, A, B, T_save)) != LBQ_OK) return st;
    const int sms = sm_count();
    const size_t need = fwd_workspace(m, q, sms, 0);
    if (need > 0 && (!workspace || workspace_bytes < need)) return LBQ_EWORKSPACE;
    if (need > 0 && !aligned16(workspace)) return LBQ_EALIGN;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    if (rank > 0) {
        if ((st = launch_lora_rows<false>(X, m, q->k, A, rank, T_save, cs)) != LBQ_OK) return st;
    }
    return run_fwd_gemm(X, m, q, B, rank, s, T_save, Y, q->n, nullptr, workspace, workspace_bytes, sms, cs);
}

lbq_status lbq_linear_fwd_noalloc(const void* X, int m, const lbq_qweight* q, const void* A, const void* B, int rank,
                                  float s, float* Y, float* T_save, lbq_stream_t stream) {
    lbq_status st = check_qweight(q, true);
    if (st != LBQ_OK) return st;
    if (m < 1 || !X || !Y) return LBQ_EINVAL;
    if (!aligned16(X) || !aligned16(Y)) return LBQ_EALIGN;
    if ((st = check_lora(rank, A, B, T_save)) != LBQ_OK) return st;
    const int sms = sm_count();
    const size_t need = fwd_workspace(m, q, sms, 0);
    if (need > kNoAllocScratchBytes) return LBQ_EWORKSPACE;  // this call's scratch does not fit
    void* scratch = nullptr;
    if ((st = noalloc_scratch_address(&scratch)) != LBQ_OK) return st;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    if (rank > 0) {
        if ((st = launch_lora_rows<false>(X, m, q->k, A, rank, T_save, cs)) != LBQ_OK) return st;
    }
    return run_fwd_gemm(X, m, q, B, rank, s, T_save, Y, q->n, nullptr, scratch, kNoAllocScratchBytes, sms, cs);
}

// Workspace of a grouped forward; ws_budget as for fwd_workspace.
static size_t grouped_fwd_workspace(int m, const lbq_fwd_problem* probs, int count, size_t ws_budget) {
    if (m < 1 || !probs || count < 1) return 0;
    const int sms = sm_count();
    if (m <= kGemvMaxM) {
        std::vector<const lbq_qweight*> qs(count);
        for (int i = 0; i < count; ++i) {
            if (check_qweight(probs[i].q, false) != LBQ_OK) return 0;
            qs[i] = probs[i].q;
        }
        return gemv_jobs_workspace(m, qs.data(), count, sms);
    }
    size_t need = 0;
    for (int i = 0; i < count; ++i) {
        if (check_qweight(probs[i].q, false) != LBQ_OK) return 0;
        need = std::max(need, plan_fwd(m, probs[i].q, sms, ws_budget).workspace());
    }
    return need;
}

size_t lbq_linear_fwd_grouped_workspace_size(int m, const lbq_fwd_problem* probs, int count) {
    return grouped_fwd_workspace(m, probs, count, ~size_t(0));
}

lbq_status lbq_linear_fwd_grouped(int m, const lbq_fwd_problem* probs, int count, void* workspace,
                                  size_t workspace_bytes, lbq_stream_t stream) {
    if (m < 1 || !probs || count < 1) return LBQ_EINVAL;
    lbq_status st;
    for (int i = 0; i < count; ++i) {
        const lbq_fwd_problem& pr = probs[i];
        if ((st = check_qweight(pr.q, true)) != LBQ_OK) return st;
        if (!pr.X || !pr.Y) return LBQ_EINVAL;
        if (!aligned16(pr.X) || !aligned16(pr.Y)) return LBQ_EALIGN;
        if ((st = check_lora(pr.rank, pr.A, pr.B, pr.T_save)) != LBQ_OK) return st;
    }
    const size_t need = grouped_fwd_workspace(m, probs, count, 0);
    if (need > 0 && (!workspace || workspace_bytes < need)) return LBQ_EWORKSPACE;
    if (need > 0 && !aligned16(workspace)) return LBQ_EALIGN;
    const int sms = sm_count();
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    for (int i = 0; i < count; ++i) {
        const lbq_fwd_problem& pr = probs[i];
        if (pr.rank > 0 && (st = launch_lora_rows<false>(pr.X, m, pr.q->k, pr.A, pr.rank, pr.T_save, cs)) != LBQ_OK)
            return st;
    }
    std::vector<GvJob> jobs(count);
    for (int i = 0; i < count; ++i) {
        const lbq_fwd_problem& pr = probs[i];
        jobs[i] = GvJob{pr.X, pr.q, pr.B, pr.rank, pr.s, pr.T_save, pr.Y, pr.q->n, nullptr};
    }
    if (m > kGemvMaxM) return run_fwd_jobs(m, jobs.data(), count, workspace, workspace_bytes, sms, cs);
    return run_gemv_jobs(m, jobs.data(), count, workspace, workspace_bytes, sms, cs);
}

// Channel-mix: the two halves in one grouped decode launch (m <= 16) or as
// two tensor-core GEMM jobs (m > 16, grouped when their tiles fill the
// machine), writing their rows' output columns through perm.
size_t lbq_linear_fwd_mix_workspace_size(int m, const lbq_qweight_mix* q, int rank) {
    (void)rank;
    if (!q || m < 1) return 0;
    if (check_qweight(&q->hi, false) != LBQ_OK || check_qweight(&q->lo, false) != LBQ_OK) return 0;
    return mix_workspace(m, q, sm_count());
}

lbq_status lbq_linear_fwd_mix(const void* X, int m, const lbq_qweight_mix* q, const void* A, const void* B, int rank,
                              float s, float* Y, float* T_save, void* workspace, size_t workspace_bytes,
                              lbq_stream_t stream) {
    lbq_status st;
    if ((st = check_mix(q, m, X, Y)) != LBQ_OK) return st;
    if ((st = check_lora(rank, A, B, T_save)) != LBQ_OK) return st;
    const int sms = sm_count();
    const size_t need = mix_workspace(m, q, sms, 0);
    if (need > 0 && (!workspace || workspace_bytes < need)) return LBQ_EWORKSPACE;
    if (need > 0 && !aligned16(workspace)) return LBQ_EALIGN;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    const int64_t n_total = static_cast<int64_t>(q->hi.n) + q->lo.n;
    if (rank > 0) {
        if ((st = launch_lora_rows<false>(X, m, q->hi.k, A, rank, T_save, cs)) != LBQ_OK) return st;
    }
    const GvJob jobs[2] = {GvJob{X, &q->hi, B, rank, s, T_save, Y, n_total, q->perm},
                           GvJob{X, &q->lo, B, rank, s, T_save, Y, n_total, q->perm + q->hi.n}};
    if (m <= kGemvMaxM) return run_gemv_jobs(m, jobs, 2, workspace, workspace_bytes, sms, cs);
    return run_fwd_jobs(m, jobs, 2, workspace, workspace_bytes, sms, cs);
}

// Workspace of a grouped channel-mix forward; ws_budget as for fwd_workspace.
static size_t mix_grouped_workspace(int m, const lbq_mix_problem* probs, int count, size_t ws_budget) {
    if (m < 1 || !probs || count < 1) return 0;
    const int sms = sm_count();
    if (m <= kGemvMaxM) {
        std::vector<const lbq_qweight*> qs;
        for (int i = 0; i < count; ++i) {
            const lbq_qweight_mix* q = probs[i].q;
            if (!q || check_qweight(&q->hi, false) != LBQ_OK || check_qweight(&q->lo, false) != LBQ_OK) return 0;
            qs.push_back(&q->hi);
            qs.push_back(&q->lo);
        }
        return gemv_jobs_workspace(m, qs.data(), static_cast<int>(qs.size()), sms);
    }
    size_t need = 0;
    for (int i = 0; i < count; ++i) {
        const lbq_qweight_mix* q = probs[i].q;
        if (!q || check_qweight(&q->hi, false) != LBQ_OK || check_qweight(&q->lo, false) != LBQ_OK) return 0;
        need = std::max(need, mix_workspace(m, q, sms, ws_budget));
    }
    return need;
}

size_t lbq_linear_fwd_mix_grouped_workspace_size(int m, const lbq_mix_problem* probs, int count) {
    return mix_grouped_workspace(m, probs, count, ~size_t(0));
}

lbq_status lbq_linear_fwd_mix_grouped(int m, const lbq_mix_problem* probs, int count, void* workspace,
                                      size_t workspace_bytes, lbq_stream_t stream) {
    if (m < 1 || !probs || count < 1) return LBQ_EINVAL;
    lbq_status st;
    for (int i = 0; i < count; ++i) {
        const lbq_mix_problem& pr = probs[i];
        if ((st = check_mix(pr.q, m, pr.X, pr.Y)) != LBQ_OK) return st;
        if ((st = check_lora(pr.rank, pr.A, pr.B, pr.T_save)) != LBQ_OK) return st;
    }
    const size_t need = mix_grouped_workspace(m, probs, count, 0);
    if (need > 0 && (!workspace || workspace_bytes < need)) return LBQ_EWORKSPACE;
    if (need > 0 && !aligned16(workspace)) return LBQ_EALIGN;
    const int sms = sm_count();
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    for (int i = 0; i < count; ++i) {
        const lbq_mix_problem& pr = probs[i];
        if (pr.rank > 0 && (st = launch_lora_rows<false>(pr.X, m, pr.q->hi.k, pr.A, pr.rank, pr.T_save, cs)) != LBQ_OK)
            return st;
    }
    std::vector<GvJob> jobs;
    for (int i = 0; i < count; ++i) {
        const lbq_mix_problem& pr = probs[i];
        const int64_t n_total = static_cast<int64_t>(pr.q->hi.n) + pr.q->lo.n;
        jobs.push_back(GvJob{pr.X, &pr.q->hi, pr.B, pr.rank, pr.s, pr.T_save, pr.Y, n_total, pr.q->perm});
        jobs.push_back(GvJob{pr.X, &pr.q->lo, pr.B, pr.rank, pr.s, pr.T_save, pr.Y, n_total, pr.q->perm + pr.q->hi.n});
    }
    if (m > kGemvMaxM) return run_fwd_jobs(m, jobs.data(), static_cast<int>(jobs.size()), workspace, workspace_bytes, sms, cs);
    return run_gemv_jobs(m, jobs.data(), static_cast<int>(jobs.size()), workspace, workspace_bytes, sms, cs);
}

size_t lbq_linear_bwd_workspace_size(int m, const lbq_qweight* q, int rank) {
    (void)rank;
    if (m < 1 || check_qweight(q, false) != LBQ_OK) return 0;
    return plan_bwd(m, q, sm_count()).workspace();
}

lbq_status lbq_linear_bwd(const void* dY, int m, const lbq_qweight* q, const void* A, const void* B, int rank,
                          float s, float* dX, float* U_save, void* workspace, size_t workspace_bytes,
                          lbq_stream_t stream) {
    lbq_status st = check_bwd(dY, m, q, A, B, rank, dX, U_save);
    if (st != LBQ_OK) return st;
    const int sms = sm_count();
    const size_t need = plan_bwd(m, q, sms, 0).workspace();
    if (need > 0 && (!workspace || workspace_bytes < need)) return LBQ_EWORKSPACE;
    if (need > 0 && !aligned16(workspace)) return LBQ_EALIGN;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    if (rank > 0) {
        if ((st = launch_lora_rows<true>(dY, m, q->n, B, rank, U_save, cs)) != LBQ_OK) return st;
    }
    return run_bwd_gemm(dY, m, q, A, rank, s, U_save, dX, workspace, workspace_bytes, sms, cs);
}

size_t lbq_linear_bwd_grouped_workspace_size(int m, const lbq_bwd_problem* probs, int count) {
    if (m < 1 || !probs || count < 1) return 0;
    const int sms = sm_count();
    size_t need = 0;
    for (int i = 0; i < count; ++i) {
        if (check_qweight(probs[i].q, false) != LBQ_OK) return 0;
        need = std::max(need, plan_bwd(m, probs[i].q, sms).workspace());
    }
    return need;
}

lbq_status lbq_linear_bwd_grouped(int m, const lbq_bwd_problem* probs, int count, void* workspace,
                                  size_t workspace_bytes, lbq_stream_t stream) {
    if (m < 1 || !probs || count < 1) return LBQ_EINVAL;
    lbq_status st;
    for (int i = 0; i < count; ++i) {
        const lbq_bwd_problem& pr = probs[i];
        if ((st = check_bwd(pr.dY, m, pr.q, pr.A, pr.B, pr.rank, pr.dX, pr.U_save)) != LBQ_OK) return st;
    }
    const int sms = sm_count();
    const int nt = std::min(token_tile(m), 256);
    const int slots = (nt >= 256 ? 1 : 2) * sms;
    int64_t tiles = 0;
    for (int i = 0; i < count; ++i) tiles += cdiv(probs[i].q->k, 128) * cdiv(m, nt);
    const bool grouped = count >= 2 && tiles >= slots;
    size_t need = 0;                                     // what the launches one by one require
    for (int i = 0; !grouped && i < count; ++i) need = std::max(need, plan_bwd(m, probs[i].q, sms, 0).workspace());
    if (need > 0 && (!workspace || workspace_bytes < need)) return LBQ_EWORKSPACE;
    if (need > 0 && !aligned16(workspace)) return LBQ_EALIGN;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    for (int i = 0; i < count; ++i) {
        const lbq_bwd_problem& pr = probs[i];
        if (pr.rank > 0 && (st = launch_lora_rows<true>(pr.dY, m, pr.q->n, pr.B, pr.rank, pr.U_save, cs)) != LBQ_OK)
            return st;
    }
    if (!grouped) {
        // too few tiles to fill the GPU together: one launch each, with its split
        for (int i = 0; i < count; ++i) {
            const lbq_bwd_problem& pr = probs[i];
            if ((st = run_bwd_gemm(pr.dY, m, pr.q, pr.A, pr.rank, pr.s, pr.U_save, pr.dX, workspace, workspace_bytes, sms,
                                   cs)) != LBQ_OK)
                return st;
        }
        return LBQ_OK;
    }
    for (int i = 0; i < count; i += kBwdMaxGroup) {
        const int c = std::min(kBwdMaxGroup, count - i);
        switch (nt) {
            case 16: st = run_bwd_group_nt<16>(m, probs + i, c, cs); break;
            case 32: st = run_bwd_group_nt<32>(m, probs + i, c, cs); break;
            case 64: st = run_bwd_group_nt<64>(m, probs + i, c, cs); break;
            case 128: st = run_bwd_group_nt<128>(m, probs + i, c, cs); break;
            default: st = run_bwd_group_nt<256>(m, probs + i, c, cs); break;
        }
        if (st != LBQ_OK) return st;
    }
    return LBQ_OK;
}

lbq_status lbq_lora_grads(const void* X, const void* dY, int m, int n, int k, const float* T, const float* U,
                          int rank, float s, float* dA, float* dB, lbq_stream_t stream) {
    if (m < 1 || n < 1 || k < 64 || k % 64 != 0 || n % 8 != 0) return LBQ_EINVAL;
    if (rank < 1 || rank > kLoraMaxRank) return LBQ_EINVAL;
    if (!X || !dY || !T || !U || !dA || !dB) return LBQ_EINVAL;
    if (!aligned16(X) || !aligned16(dY) || !aligned16(T) || !aligned16(U) || !aligned16(dA) || !aligned16(dB))
        return LBQ_EALIGN;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    lbq_status st = launch_lora_colgrad(X, m, k, U, rank, s, dA, 1, k, cs);
    if (st != LBQ_OK) return st;
    return launch_lora_colgrad(dY, m, n, T, rank, s, dB, rank, 1, cs);
}

#ifdef LBQ_TRACE
// Trace builds only: copy the pipeline trace (kinds x 256 clock stamps).
int lbq_trace_read(long long* host, int n) {
    const int total = kTraceKinds * kTraceLen;
    if (cudaDeviceSynchronize() != cudaSuccess) return -1;
    if (cudaMemcpyFromSymbol(host, g_trace, sizeof(long long) * (n < total ? n : total)) != cudaSuccess) return -1;
    return total;
}
#endif

size_t lbq_channel_mix_select_workspace_size(int n, int k) {
    if (n < 1 || k < 128) return 0;
    return round_up(static_cast<size_t>(k) * sizeof(double), 256) + round_up(static_cast<size_t>(n) * sizeof(double), 256) +
           round_up(static_cast<size_t>(n), 256);
}

lbq_status lbq_channel_mix_select(const void* W_bf16, int n, int k, const void* X_bf16, int t, int n4, double* score,
                                  int32_t* perm, void* workspace, size_t workspace_bytes, lbq_stream_t stream) {
    if (!W_bf16 || !X_bf16 || !perm || n < 1 || k < 128 || k % 128 != 0 || t < 1 || n4 < 0 || n4 > n)
        return LBQ_EINVAL;
    if (!aligned16(W_bf16) || !aligned16(X_bf16) || !aligned16(perm) || (score && !aligned16(score)))
        return LBQ_EALIGN;
    const size_t need = lbq_channel_mix_select_workspace_size(n, k);
    if (!workspace || workspace_bytes < need) return LBQ_EWORKSPACE;
    if (!aligned16(workspace)) return LBQ_EALIGN;
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    double* m2 = reinterpret_cast<double*>(ws);
    double* sc = reinterpret_cast<double*>(ws + round_up(static_cast<size_t>(k) * sizeof(double), 256));
    uint8_t* sel = ws + round_up(static_cast<size_t>(k) * sizeof(double), 256) +
                   round_up(static_cast<size_t>(n) * sizeof(double), 256);
    if (score) sc = score;
    second_moment_kernel<<<static_cast<unsigned>(cdiv(k, 256)), 256, 0, cs>>>(static_cast<const uint16_t*>(X_bf16), t,
                                                                             k, m2);
    lbq_status st = last_launch();
    if (st != LBQ_OK) return st;
    channel_score_kernel<<<static_cast<unsigned>(cdiv(n, 8)), 256, 0, cs>>>(static_cast<const uint16_t*>(W_bf16), n, k,
                                                                          m2, sc);
    if ((st = last_launch()) != LBQ_OK) return st;
    channel_rank_kernel<<<static_cast<unsigned>(cdiv(n, 256)), 256, 0, cs>>>(sc, n, n4, sel);
    if ((st = last_launch()) != LBQ_OK) return st;
    channel_perm_kernel<<<1, 1024, 0, cs>>>(sel, n, n4, perm);
    return last_launch();
}

lbq_status lbq_gather_rows(const void* W_bf16, int n, int k, const int32_t* rows, int count, void* out,
                           lbq_stream_t stream) {
    if (!W_bf16 || !rows || !out || n < 1 || k < 8 || k % 8 != 0 || count < 1) return LBQ_EINVAL;
    if (!aligned16(W_bf16) || !aligned16(out)) return LBQ_EALIGN;
    const int64_t total = static_cast<int64_t>(count) * (k / 8);
    const int grid = static_cast<int>(std::min<int64_t>(cdiv(total, 256), 16LL * sm_count()));
    gather_rows_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4*>(W_bf16), k / 8, rows, count, static_cast<uint4*>(out));
    return last_launch();
}

lbq_status lbq_linear_fwd_noalloc_reset(lbq_stream_t stream) {
    void* scratch = nullptr;
    lbq_status st = noalloc_scratch_address(&scratch);
    if (st != LBQ_OK) return st;
    return cudaMemsetAsync(scratch, 0, kCounterHeader, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
               ? LBQ_OK
               : LBQ_ECUDA;
}

lbq_status lbq_selftest_wait_timeout(uint32_t limit_us, lbq_stream_t stream) {
    if (limit_us < 1 || limit_us > 1000000u) return LBQ_EINVAL;
    wait_timeout_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(uint64_t(limit_us) * 1000u);
    return last_launch();
}

lbq_status lbq_device_status(uint32_t* flags) {
    if (!flags) return LBQ_EINVAL;
    if (cudaDeviceSynchronize() != cudaSuccess) return LBQ_ECUDA;
    uint32_t v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_status, sizeof(v)) != cudaSuccess) return LBQ_ECUDA;
    if (cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess) return LBQ_ECUDA;
    *flags = v;
    return LBQ_OK;
}

}  // extern "C"
