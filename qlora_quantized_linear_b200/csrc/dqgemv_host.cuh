// dqgemv_host.cuh -- host side of the decode GEMV: shared-memory budget,
// stream-K plan (shares, grid, weight-ring depth) and the launch.  Included by
// lbq.cu inside its file-local namespace, after the plan type, workspace
// layout and stream bookkeeping it uses.
#pragma once

// Decode-sized batches (m <= 16) run the stream-K GEMV: every CTA gets an
// equal share of the (row tile, k-block) work, a whole number of scale
// groups and as many k-blocks as its shared memory holds (weight ring,
// activation slice, constant table) with two CTAs per SM, and the grid fills
// whole waves of two CTAs per SM.  The weight ring holds four boxes, or
// three when that lets the whole grid run in one wave (wide token tiles,
// whose activation slice takes most of the shared memory).
constexpr int kGemvMaxM = 16;
constexpr size_t kGemvSmemBudget = 113 * 1024;     // two CTAs per SM

size_t gemv_smem_bytes(int m, int share, int kind, int stages) {
    const int gb = kind == kInt4 ? 2 : 1;
    const int nt = m <= 8 ? 8 : 16;
    const size_t xrows = static_cast<size_t>(m < nt ? m + 1 : m);      // + a zero row for padded lanes
    return 1024 + static_cast<size_t>(stages) * 128 * 128 + xrows * (share * 64 + 4) * 2 +
           static_cast<size_t>((share / gb) | 1) * 128 * 4 + (kind == kCode4 ? 1024 : 0) + 2 * stages * 8 + 16;
}

Plan plan_gemv(int m, const lbq_qweight* q, int sms) {
    Plan pl;
    pl.nt = m <= 8 ? 8 : 16;
    const int kind = kind_of(q);
    const int64_t kbt = q->k / 64;
    const int gb = kind == kInt4 ? 2 : 1;
    pl.tiles = static_cast<int>(cdiv(q->n, 128));
    const int64_t total = static_cast<int64_t>(pl.tiles) * kbt;
    const int64_t slots = 2LL * sms;
    auto max_share = [&](int stages) {
        int64_t smax = gb;
        while (smax + gb <= kbt && (smax + gb) / gb <= kGemvMaxTabGroups &&
               gemv_smem_bytes(m, static_cast<int>(smax + gb), kind, stages) <= kGemvSmemBudget)
            smax += gb;
        return smax;
    };
    int64_t smax = max_share(kGemvMaxWStages);
    int64_t waves = cdiv(total, slots * smax);
    pl.stages = kGemvMaxWStages;
    if (waves > 1) {
        const int64_t smax3 = max_share(kGemvMaxWStages - 1);
        if (cdiv(total, slots * smax3) < waves) {
            smax = smax3;
            waves = cdiv(total, slots * smax3);
            pl.stages = kGemvMaxWStages - 1;
        }
    }
    int64_t share = cdiv(cdiv(total, waves * slots), gb) * gb;
    // at least an eighth of a row per CTA, so that the CTA finishing a tile
    // sums a handful of partials (small layers then use fewer CTAs)
    share = std::max(share, std::min(cdiv(cdiv(kbt, 8), gb) * gb, smax));
    share = std::max<int64_t>(gb, std::min(share, smax));
    pl.per_split = static_cast<int>(share);                      // k-blocks per CTA
    pl.nsplit = static_cast<int>(cdiv(total, share));            // CTAs
    pl.partial_bytes = round_up(static_cast<size_t>(pl.nsplit + pl.tiles) * m * 128 * sizeof(float), 256);
    return pl;
}

template <int KIND, int NTOK, int WS>
lbq_status launch_gemv_kind(const GemvParams& p, const uint8_t* packed, int grid, cudaStream_t st) {
    auto kern = dqgemv_kernel<KIND, NTOK, WS>;
    const size_t smem = gemv_smem_bytes(p.m, p.share, KIND, WS);
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
        return LBQ_ECUDA;
    CUtensorMap tmW;
    if (!make_map_2d(&tmW, packed, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, p.n, static_cast<int64_t>(p.k) * (KIND == kInt2 ? 2 : 4) / 8,
                     128, 128, CU_TENSOR_MAP_SWIZZLE_128B))
        return LBQ_ECUDA;
    // programmatic dependent launch: the kernel may start during the previous
    // kernel's tail and waits for it (griddepcontrol.wait) before reading
    // anything that kernel can have written
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
    cfg.blockDim = dim3(kGemvThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, tmW, p) != cudaSuccess) return LBQ_ECUDA;
    return last_launch();
}

template <int WS>
lbq_status launch_gemv_tile(const GemvParams& p, const lbq_qweight* q, const Plan& pl, cudaStream_t st) {
    if (WS != pl.stages) {
        if constexpr (WS > kGemvMaxWStages - 1) return launch_gemv_tile<WS - 1>(p, q, pl, st);
        return LBQ_EUNSUPPORTED;
    }
    const bool n8 = pl.nt == 8;
    switch (kind_of(q)) {
        case kInt4: return n8 ? launch_gemv_kind<kInt4, 8, WS>(p, q->packed, pl.nsplit, st)
                              : launch_gemv_kind<kInt4, 16, WS>(p, q->packed, pl.nsplit, st);
        case kInt2: return n8 ? launch_gemv_kind<kInt2, 8, WS>(p, q->packed, pl.nsplit, st)
                              : launch_gemv_kind<kInt2, 16, WS>(p, q->packed, pl.nsplit, st);
        default: return n8 ? launch_gemv_kind<kCode4, 8, WS>(p, q->packed, pl.nsplit, st)
                           : launch_gemv_kind<kCode4, 16, WS>(p, q->packed, pl.nsplit, st);
    }
}

// One fused dequantize-GEMM over one stored weight (or one half of a
// channel-mix weight).  `perm` maps its stored rows to output columns.
lbq_status run_gemv(const void* X, int m, const lbq_qweight* q, const void* B, int rank, float s, const float* T,
                    float* Y, int64_t ldy, const int32_t* perm, void* ws, int sms, cudaStream_t st) {
    const Plan pl = plan_gemv(m, q, sms);
    GemvParams p{};
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
    p.X = static_cast<const uint16_t*>(X);
    p.rank = rank;
    p.s = s;
    p.T = T;
    p.B = static_cast<const uint16_t*>(B);
    p.Y = Y;
    p.ldy = ldy;
    p.perm = perm;
    p.kbt = q->k / 64;
    p.tiles = pl.tiles;
    p.share = pl.per_split;
    p.total = static_cast<int64_t>(pl.tiles) * p.kbt;
    p.w_early = weights_stable(st) ? 1 : 0;
    if (p.total >= (int64_t(1) << 31)) return LBQ_EUNSUPPORTED;
    if (pl.workspace() > 0) {
        if (!ws) return LBQ_EWORKSPACE;
        if (pl.tiles > kMaxSplitTiles) return LBQ_EUNSUPPORTED;
        p.partial = ws_partials(ws);
        p.counters = ws_counters(ws);
    }
    return launch_gemv_tile<4>(p, q, pl, st);
}
