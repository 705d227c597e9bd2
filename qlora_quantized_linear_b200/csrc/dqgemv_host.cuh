// dqgemv_host.cuh -- host side of the grouped decode GEMV: shared-memory
// layout, shares and grid, workspace layout and the launch.  Included by
// lbq.cu inside its file-local namespace, after the helpers it uses (tensor
// maps, descriptor checks, workspace header, stream bookkeeping).
#pragma once

// Decode-sized batches (m <= 16) run the grouped GEMV: one launch for up to
// kGvMaxProblems matrices, one wave of two CTAs per SM, every CTA an equal
// share in bytes of one matrix's (row tile, k-block) work.
constexpr int kGemvMaxM = 16;
constexpr size_t kGemvSmemBudget = 115712 - 1024;   // two CTAs per SM (228 KB; 1 KB reserved and 1 KB static per CTA)

// One forward of a group: activations, weight, adapter, output.
struct GvJob {
    const void* X;
    const lbq_qweight* q;
    const void* B;
    int rank;
    float s;
    const float* T;
    float* Y;
    int64_t ldy;
    const int32_t* perm;
};

struct GvPlan {
    int count = 0;
    int ctas = 0;                   // grid
    int ws = 0;                     // ring stages
    int stage_bytes = 0, xbox_max = 0, cstride = 0;
    size_t smem = 0;                // dynamic shared memory per CTA
    size_t workspace = 0;           // 0 when no tile is split
    int share[kGvMaxProblems] = {}, pctas[kGvMaxProblems] = {}, cta0[kGvMaxProblems] = {};
    int tiles[kGvMaxProblems] = {};
    int cnt_off[kGvMaxProblems] = {};
    size_t part_off[kGvMaxProblems] = {};
};

// Algorithmic bytes of one (128-row tile, k-block) unit: packed codes plus
// the per-row constants of the k-block.
double gv_unit_bytes(const lbq_qweight* q) {
    const double codes = 128.0 * 64 * q->bits / 8;
    if (q->scheme == LBQ_MINMAX_ASYM) return codes + 128.0 * 4 * 64 / q->group;
    return codes + 128.0 * (q->double_quant ? 1 : 4);
}

// Bytes per row of one constant array that a compute warp's part of a weight
// box needs (half the box's k-blocks with up to 8 tokens, all of them with
// more): the 4-byte words covering its groups (MinMax, starting at any
// entry), its absmax values, or 2 words of q8 (and of s2 in the second array).
int gv_const_stride(const lbq_qweight* q, int m) {
    const int parts = m <= 8 ? 2 : 1;
    const int kpp = (q->scheme == LBQ_MINMAX_ASYM && q->bits == 2 ? 8 : 4) / parts;   // k-blocks per part
    if (q->scheme == LBQ_CODEBOOK4) return q->double_quant ? 8 : 4 * kpp;
    const int gpp = q->bits == 2 ? kpp : kpp / 2;                                    // groups per part
    return 4 * (gpp / 2 + 1);
}

// Token rows of an activation box: the real ones padded to the MMA's token
// tile (8 or 16).
int gv_mpad(int m) { return m <= 8 ? 8 : 16; }

lbq_status gv_plan(int m, const lbq_qweight* const* qs, int count, int sms, GvPlan* pl) {
    if (m < 1 || m > kGemvMaxM || count < 1 || count > kGvMaxProblems) return LBQ_EINVAL;
    *pl = GvPlan();
    pl->count = count;
    bool any_int2 = false, any_code = false;
    int cstride = 4;
    double total_bytes = 0.0;
    int tiles_sum = 0;
    for (int i = 0; i < count; ++i) {
        const lbq_qweight* q = qs[i];
        const int64_t kbt = q->k / 64, tiles = cdiv(q->n, 128);
        if (tiles * kbt >= (int64_t(1) << 31)) return LBQ_EUNSUPPORTED;
        any_int2 |= (q->scheme == LBQ_MINMAX_ASYM && q->bits == 2);
        any_code |= q->scheme == LBQ_CODEBOOK4;
        cstride = std::max(cstride, gv_const_stride(q, m));
        total_bytes += gv_unit_bytes(q) * static_cast<double>(tiles * kbt);
        pl->tiles[i] = static_cast<int>(tiles);
        pl->cnt_off[i] = tiles_sum;
        tiles_sum += static_cast<int>(tiles);
    }
    if (tiles_sum > kMaxSplitTiles) return LBQ_EUNSUPPORTED;
    // stage layout: weight box, activation box; after the ring each compute
    // warp's constant double buffer ([2 slots][2 arrays][its 32 or 16 rows]
    // [cstride]) and the buffer in which the compute warps add the two
    // k-halves of their rows
    const int sub_max = any_int2 ? 8 : 4;
    pl->xbox_max = sub_max * gv_mpad(m) * 128;
    pl->cstride = cstride;
    pl->stage_bytes = kGvWBox + pl->xbox_max;
    const size_t cbuf = static_cast<size_t>(kGvComputeWarps) * 2 * 2 * (m <= 8 ? 32 : 16) * cstride;
    const size_t xchg = m <= 8 ? kGvXchgBytes : 0;
    (void)any_code;
    pl->ws = 0;
    for (int ws = kGvMaxStages; ws >= 2; --ws) {
        const size_t smem = 1024 + static_cast<size_t>(ws) * pl->stage_bytes + cbuf + xchg + kGvExtraSmem;
        if (smem <= kGemvSmemBudget) {
            pl->ws = ws;
            pl->smem = smem;
            break;
        }
    }
    if (pl->ws == 0) return LBQ_EUNSUPPORTED;
    // shares: every CTA about the same bytes; at most one wave of two CTAs
    // per SM (each matrix rounds its CTA count up by less than one)
    const int slots = 2 * sms;
    const double target = total_bytes / std::max(1, slots - count);
    bool split = false;
    size_t part = 0;
    int cta = 0;
    for (int i = 0; i < count; ++i) {
        const lbq_qweight* q = qs[i];
        const int64_t kbt = q->k / 64, units = static_cast<int64_t>(pl->tiles[i]) * kbt;
        const int gb = (q->scheme == LBQ_MINMAX_ASYM && q->bits == 4) ? 2 : 1;
        int64_t share = cdiv(static_cast<int64_t>(std::ceil(target / gv_unit_bytes(q))), gb) * gb;
        // at least an eighth of a row per CTA, so that the CTA finishing a
        // tile sums a handful of partials (small matrices use fewer CTAs)
        share = std::max(share, std::min<int64_t>(kbt, cdiv(cdiv(kbt, 8), gb) * gb));
        share = std::max<int64_t>(share, gb);
        const int64_t ctas = cdiv(units, share);
        pl->share[i] = static_cast<int>(share);
        pl->pctas[i] = static_cast<int>(ctas);
        pl->cta0[i] = cta;
        cta += static_cast<int>(ctas);
        if (share % kbt != 0) split = true;
        pl->part_off[i] = part;
        part += round_up(static_cast<size_t>(ctas + pl->tiles[i]) * m * 128 * sizeof(float), 256);
    }
    pl->ctas = cta;
    pl->workspace = split ? kCounterHeader + part : 0;
    return LBQ_OK;
}

template <int NT8>
lbq_status gv_launch(const GvParams& prm, const GvPlan& pl, cudaStream_t st) {
    auto kern = dqgemv_grouped_kernel<NT8>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(pl.smem)) != cudaSuccess)
        return LBQ_ECUDA;
    // programmatic dependent launch: the kernel may start during the previous
    // kernel's tail and waits for it (griddepcontrol.wait) before reading
    // anything that kernel can have written
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(pl.ctas), 1, 1);
    cfg.blockDim = dim3(kGvThreads, 1, 1);
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, prm) != cudaSuccess) return LBQ_ECUDA;
    return last_launch();
}

// One grouped launch (count <= kGvMaxProblems) of the decode GEMV.
lbq_status run_gemv_group(int m, const GvJob* jobs, int count, void* ws, size_t ws_bytes, int sms, cudaStream_t st) {
    const lbq_qweight* qs[kGvMaxProblems];
    for (int i = 0; i < count; ++i) qs[i] = jobs[i].q;
    GvPlan pl;
    lbq_status s = gv_plan(m, qs, count, sms, &pl);
    if (s != LBQ_OK) return s;
    if (pl.workspace > 0 && (!ws || ws_bytes < pl.workspace)) return LBQ_EWORKSPACE;
    GvParams prm;                                // passed by value at launch
    memset(&prm, 0, sizeof(prm));
    prm.nprob = count;
    prm.m = m;
    prm.ws = pl.ws;
    prm.stage_bytes = pl.stage_bytes;
    prm.cstride = pl.cstride;
    prm.w_early = weights_stable(st) ? 1 : 0;
    for (int i = 0; i < count; ++i) {
        const lbq_qweight* q = jobs[i].q;
        GvProblem& P = prm.prob[i];
        const int sub = (q->scheme == LBQ_MINMAX_ASYM && q->bits == 2) ? 8 : 4;
        if (!make_map_2d(&prm.tmW[i], q->packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, q->n,
                         static_cast<int64_t>(q->k) * q->bits / 8, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B))
            return LBQ_ECUDA;
        if (!make_map_x3d(&prm.tmX[i], jobs[i].X, m, q->k, gv_mpad(m), sub)) return LBQ_ECUDA;
        P.xbytes = sub * gv_mpad(m) * 128;
        P.X = static_cast<const uint16_t*>(jobs[i].X);
        P.Y = jobs[i].Y;
        P.perm = jobs[i].perm;
        P.scale = q->scale;
        P.zero = q->zero;
        P.absmax = q->absmax;
        P.q8 = (q->scheme == LBQ_CODEBOOK4 && q->double_quant) ? q->absmax_q8 : nullptr;
        P.s2 = q->absmax_s2;
        P.offset = q->absmax_offset;
        P.codebook = q->codebook;
        P.T = jobs[i].T;
        P.B = static_cast<const uint16_t*>(jobs[i].B);
        P.rank = jobs[i].rank;
        P.s = jobs[i].s;
        P.ldy = jobs[i].ldy;
        P.n = q->n;
        P.k = q->k;
        P.kind = kind_of(q);
        P.ngroups = q->scheme == LBQ_MINMAX_ASYM ? q->k / q->group : 0;
        P.kbt = q->k / 64;
        P.tiles = pl.tiles[i];
        P.total = static_cast<int64_t>(pl.tiles[i]) * P.kbt;
        P.share = pl.share[i];
        P.cta0 = pl.cta0[i];
        if (pl.workspace > 0) {
            P.counters = ws_counters(ws) + pl.cnt_off[i];
            P.partial = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(ws_partials(ws)) + pl.part_off[i]);
        }
    }
    return m <= 8 ? gv_launch<1>(prm, pl, st) : gv_launch<2>(prm, pl, st);
}

// Any number of matrices: groups of kGvMaxProblems, one launch each, in order.
lbq_status run_gemv_jobs(int m, const GvJob* jobs, int count, void* ws, size_t ws_bytes, int sms, cudaStream_t st) {
    for (int i = 0; i < count; i += kGvMaxProblems) {
        const lbq_status s = run_gemv_group(m, jobs + i, std::min(kGvMaxProblems, count - i), ws, ws_bytes, sms, st);
        if (s != LBQ_OK) return s;
    }
    return LBQ_OK;
}

// Workspace of run_gemv_jobs: the largest of its launches'.
size_t gemv_jobs_workspace(int m, const lbq_qweight* const* qs, int count, int sms) {
    size_t need = 0;
    for (int i = 0; i < count; i += kGvMaxProblems) {
        GvPlan pl;
        if (gv_plan(m, qs + i, std::min(kGvMaxProblems, count - i), sms, &pl) == LBQ_OK)
            need = std::max(need, pl.workspace);
    }
    return need;
}
