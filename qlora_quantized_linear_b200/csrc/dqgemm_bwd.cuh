// dqgemm_bwd.cuh -- input gradient through the frozen quantized weight on the
// 5th-generation tensor cores (QLoRA explainer, QLoRA技术原理: gradients flow
// through the frozen 4-bit weight into the adapters):
//
//   dX[t, k] = sum_c dY[t, c] * W_hat[c, k]  (+ s * sum_u U[t, u] A[u, k])
//
// computed as dX^T = W_hat^T dY^T: one CTA owns 128 input features x NT tokens
// and runs over the output channels c in blocks of 64.
//
//  * The weight is read in its stored [n, k] packed layout.  Each block's
//    64 channel rows x 128 features are dequantized row-wise -- the same cheap
//    per-word unpacking as the forward -- into a bf16 tile in shared memory
//    laid out as the MMA's A operand in MN-major form (features contiguous,
//    128-byte swizzle).  No column gathers, no transposed copy.
//  * dY tiles [NT tokens x 64 channels] arrive by TMA as the K-major B operand.
//  * tcgen05.mma (A and B from shared memory, fp32 accumulator in tensor
//    memory) computes D[feature, token].
//  * Codes are paired as in the forward (two codes of a 32-bit word that sit
//    two bytes apart), so within every 8 (INT4) or 16 (INT2) features the A
//    tile holds the features in a fixed permuted order; the epilogue writes
//    each tensor-memory lane back to its own feature.
//  * Roles: warp 0 TMA producer, warp 1 TMEM owner and MMA issuer, then 16
//    (256-token tile) or 8 warps dequantize and run the epilogue.  Rings, bounded waits and the split-K
//    reduction (the last CTA of a tile sums the partials in split order) follow
//    the forward kernel.
#pragma once

#include "dqgemm.cuh"
#include "dqgemv.cuh"

namespace lbq {

// Order of the 8 (4-bit) or 16 (2-bit) features of a pairing group as the
// dequantized tile holds them: 4-bit codes pair nibbles two bytes apart
// (features k and k+4 of a word), 2-bit codes pair crumbs two bytes apart
// (k and k+8).  Entry p is the feature stored at position p.
__device__ __forceinline__ int bwd_xperm(int kind, int p) {
    constexpr int kPerm4[16] = {1, 5, 0, 4, 3, 7, 2, 6, 9, 13, 8, 12, 11, 15, 10, 14};
    constexpr int kPerm2[16] = {0, 8, 1, 9, 2, 10, 3, 11, 4, 12, 5, 13, 6, 14, 7, 15};
    return kind == kInt2 ? kPerm2[p] : kPerm4[p];
}

struct BwdParams {
    int m, n, k;                 // tokens, weight rows (output channels), input features
    int bits, ngroups, group;    // MinMax bit width, k / group, group
    const uint16_t* scale;       // [n, ngroups]
    const uint16_t* zero;        // [n, ngroups]
    const float* absmax;         // [n * k / 64] (codebook, no double quant)
    const int8_t* q8;            // [n * k / 64] (codebook, double quant)
    const float* s2;             // [ceil(n * k / 64 / 256)]
    const float* offset;         // [1]
    const float* codebook;       // [16]
    int rank, rank_pad;
    float s;
    const float* U;              // [m, rank] fp32
    const uint16_t* A;           // [rank, k] bf16
    float* dX;                   // [m, k]
    int cb_per_split;            // blocks of 64 output channels per split
    int nsplit;                  // splits of every tile of this launch
    int tile0;                   // first tile of this launch (tiles numbered feature tile fastest)
    int ftiles;                  // 128-feature tiles of the GEMM
    float* partial;              // [tile - tile0][nsplit][NT tokens][128 lanes] fp32 (nsplit > 1)
    uint32_t* counters;
};


template <int NT>
struct BwdCfg {
    static constexpr int kXStages = NT <= 64 ? 4 : NT <= 128 ? 2 : 4;   // dY tiles in flight (see the forward)
    static constexpr int kWStages = 4;
    static constexpr int kAStages = NT <= 64 ? 3 : NT >= 256 ? 3 : 2;
    static constexpr int kMinBlocks = NT >= 256 ? 1 : 2;   // CTAs per SM
    static constexpr int kDqWarps = NT >= 256 ? 16 : 8;     // dequantize + epilogue warps
};

template <int NT, int BITS, int XS, int WS, int AS>
struct BwdSmem {
    static constexpr int kKTB = 128 * BITS / 8;      // packed bytes of one channel row across the tile
    static constexpr int kXBytes = NT * 128;         // dY tile: NT tokens x 64 channels, bf16
    static constexpr int kWBytes = 64 * kKTB;        // packed weight tile: 64 channels
    static constexpr int kABytes = 64 * 128 * 2;     // A tile: 64 channels x 128 features, bf16
    static constexpr size_t kX = 0;                  // all SW128 tiles 1024-byte aligned
    static constexpr size_t kA = kX + size_t(XS) * kXBytes;
    static constexpr size_t kW = kA + size_t(AS) * kABytes;
    static constexpr size_t kBar = kW + size_t(WS) * kWBytes;
    static constexpr int kNumBars = 2 * XS + 2 * WS + 2 * AS + 1;
    static constexpr size_t kMisc = kBar + kNumBars * 8;
    static constexpr size_t kLoraT = (kMisc + 128 + 1023) / 1024 * 1024;   // s*U operand tile
    static size_t total(int rank) { return kLoraT + (rank > 0 ? size_t(NT) * 128 : 0) + 1024; }
};

// Shared-memory descriptor of an MN-major operand with the 128-byte swizzle:
// atoms of 8 K-rows x 128 bytes, `lbo` bytes between atoms along M (or N),
// `sbo` bytes between groups of 8 K-rows.
__device__ __forceinline__ uint64_t smem_desc_mn_sw128(uint32_t smem_addr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
    d |= static_cast<uint64_t>(1u) << 46;
    d |= static_cast<uint64_t>(2u) << 61;
    return d;
}

// D (tensor memory) [+]= A (shared, descriptor) * B (shared, descriptor).
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Byte offset of 16-byte unit `fu` (features 8 fu .. 8 fu + 7) of channel row
// c (0..63) in the MN-major A tile [64 channels][128 features]: groups of 8
// channels 2048 bytes apart, the two 64-feature halves 1024 bytes apart,
// rows 128 bytes apart, units swizzled with the row.
__device__ __forceinline__ uint32_t bwd_a_offset(int c, int fu) {
    const int row = c & 7, uu = fu & 7;
    return static_cast<uint32_t>((c >> 3) * 2048 + (fu >> 3) * 1024 + row * 128 + ((uu ^ row) << 4));
}

// The output tile a CTA computes: features k0 .. k0 + 127, tokens t0 ..
// t0 + NT - 1, channel split `split`; `tile` numbers the tile within its
// GEMM (the split counters).
struct BwdTile {
    int k0, t0, split;
    uint32_t tile;
};

// One CTA of the backward GEMM; tmDY and tmW are the tensor maps of dY and
// of the packed weight.
template <int NT, int KIND, int XS, int WS, int AS, int DQW>
__device__ __forceinline__ void bwd_tile(const CUtensorMap* tmDY, const CUtensorMap* tmW, const BwdParams& p,
                                         const BwdTile tl) {
    constexpr int BITS = KIND == kInt2 ? 2 : 4;
    using L = BwdSmem<NT, BITS, XS, WS, AS>;
    constexpr int KTB = L::kKTB;
    constexpr int PG = BITS == 4 ? 8 : 16;                 // features per pairing group
    constexpr int WPR = BITS == 4 ? 16 : 8;                // 32-bit code words per channel row of a block
    constexpr int SLOTS = 64 * WPR / (32 * DQW);           // (channel, word) units per thread and block
    constexpr int PARTS = DQW / 4;                         // epilogue warps per TMEM lane quarter
    constexpr uint32_t kTmemCols = tmem_cols_for(NT);
    constexpr uint32_t kIdesc = idesc_bf16_f32(128, NT) | (1u << 15);   // A is MN-major

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* sX = smem + L::kX;
    uint8_t* sA = smem + L::kA;
    uint8_t* sW = smem + L::kW;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
    uint64_t* fullX = bars;
    uint64_t* emptyX = fullX + XS;
    uint64_t* fullW = emptyX + XS;
    uint64_t* emptyW = fullW + WS;
    uint64_t* afull = emptyW + WS;
    uint64_t* aempty = afull + AS;
    uint64_t* dfull = aempty + AS;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + L::kMisc);
    volatile int* s_abort = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
    int* s_last = reinterpret_cast<int*>(smem + L::kMisc + 8);
    float* s_cb = reinterpret_cast<float*>(smem + L::kMisc + 64);   // codebook, 16 floats
    uint8_t* sUop = smem + L::kLoraT;                  // s*U operand tile [NT x 128 B] (bf16, K-major, SW128)

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int k0 = tl.k0;
    const int t0 = tl.t0;
    const int split = tl.split;
    const int cb_total = (p.n + 63) / 64;
    const int cb0 = split * p.cb_per_split;
    const int ncb = min(p.cb_per_split, cb_total - cb0);
    // The token tiles start their walk over the channel blocks at different
    // blocks (a fixed rotation per token tile), so that a block's scales and
    // zeros are not first requested by all CTAs of a wave at once, while the
    // CTAs of one token tile, which read the same dY tiles, walk together;
    // the order of the sum over blocks is then fixed per tile.
    const int rot = ncb > 0 ? static_cast<int>((static_cast<int64_t>(t0 / NT) * 37) % ncb) : 0;
    auto blk = [&](int i) { return cb0 + (i + rot < ncb ? i + rot : i + rot - ncb); };
    // the adapter term s * U A enters the accumulator through rank/16 MMAs
    // before the main loop, in the first split only; its A operand (the rows
    // of A) takes the first slot of the A ring, as a block before the first
    const bool lora = p.rank > 0 && split == 0;
    const int a_off = lora ? 1 : 0;

    if (threadIdx.x == 0) {
        for (int i = 0; i < XS; ++i) {
            mbar_init(&fullX[i], 1);
            mbar_init(&emptyX[i], 1);
        }
        for (int i = 0; i < WS; ++i) {
            mbar_init(&fullW[i], 1);
            mbar_init(&emptyW[i], DQW);
        }
        for (int i = 0; i < AS; ++i) {
            mbar_init(&afull[i], DQW);
            mbar_init(&aempty[i], 1);
        }
        mbar_init(dfull, 1);
        *s_abort = 0;
        fence_mbar_init();
    }
    if (KIND == kCode4 && threadIdx.x < 16) s_cb[threadIdx.x] = p.codebook[threadIdx.x];
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(tmDY);
        tma_prefetch_desc(tmW);
    }
    if (warp == 1) {
        tmem_alloc(s_tmem, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *s_tmem;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            // two independent streams, each issued as soon as its ring has a
            // free slot (weights: released by the dequantize warps; dY: by
            // the MMAs)
            int wi = 0, xi = 0;
            ProgressGuard guard;
            bool ok = true;
            while (ok && (wi < ncb || xi < ncb)) {
                bool prog = false;
                if (wi < ncb && (wi < WS || mbar_try_wait(&emptyW[wi % WS], ((wi / WS) - 1) & 1))) {
                    const int w = wi % WS;
                    mbar_arrive_expect_tx(&fullW[w], L::kWBytes);
                    tma_load_2d(sW + w * L::kWBytes, tmW, &fullW[w], k0 * BITS / 8, blk(wi) * 64);
                    ++wi;
                    prog = true;
                }
                if (xi < ncb && (xi < XS || mbar_try_wait(&emptyX[xi % XS], ((xi / XS) - 1) & 1))) {
                    const int x = xi % XS;
                    mbar_arrive_expect_tx(&fullX[x], L::kXBytes);
                    tma_load_2d(sX + x * L::kXBytes, tmDY, &fullX[x], blk(xi) * 64, t0);
                    ++xi;
                    prog = true;
                }
                ok = guard.step(prog, s_abort);
            }
            for (int i = max(0, xi - XS); i < xi; ++i) mbar_wait_drain(&fullX[i % XS], (i / XS) & 1);
            for (int i = max(0, wi - WS); i < wi; ++i) mbar_wait_drain(&fullW[i % WS], (i / WS) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            bool ok = true;
            if (lora) {
                // D = A^T (s U)^T: A operand = the adapter's A rows (A ring slot 0), B operand = s U
                ok = mbar_wait(&afull[0], 0, s_abort);
                tc_fence_after();
                const uint32_t abase = smem_u32(sA);
                const uint64_t udesc = smem_desc_k_sw128(smem_u32(sUop));
                for (int j = 0; ok && j < p.rank_pad / 16; ++j)
                    mma_ss(tmem, smem_desc_mn_sw128(abase + j * 4096, 1024, 2048), udesc + static_cast<uint64_t>(2 * j),
                           kIdesc, j > 0 ? 1u : 0u);
                if (ok) mma_commit(&aempty[0]);
            }
            for (int i = 0; i < ncb && ok; ++i) {
                const int x = i % XS, ia = i + a_off, a = ia % AS;
                ok = mbar_wait(&fullX[x], (i / XS) & 1, s_abort) && mbar_wait(&afull[a], (ia / AS) & 1, s_abort);
                if (!ok) break;
                tc_fence_after();
                const uint32_t abase = smem_u32(sA + a * L::kABytes);
                const uint64_t bdesc = smem_desc_k_sw128(smem_u32(sX + x * L::kXBytes));
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    mma_ss(tmem, smem_desc_mn_sw128(abase + j * 4096, 1024, 2048), bdesc + static_cast<uint64_t>(2 * j),
                           kIdesc, (lora || i > 0 || j > 0) ? 1u : 0u);
                mma_commit(&emptyX[x]);
                mma_commit(&aempty[a]);
            }
            mma_commit(dfull);          // also completes when nothing was issued
            mbar_wait_drain(dfull, 0);  // MMAs done before tensor memory is freed
        }
    } else {
        // ------------------------------------------------------------ dequantize
        const int tid = threadIdx.x - 64;                  // 0 .. 32 DQW - 1
        // unit slot u: channel row cl(u) of the block and word fw of that row
        const int fw = tid % WPR;
        const int crow0 = tid / WPR;
        constexpr int cstep = 32 * DQW / WPR;
        const int gsub = BITS == 4 ? 0 : (fw >> 2);        // 64-feature group of this word (INT2 g64)
        const int gcol = KIND == kCode4 ? 0 : k0 / p.group + gsub;
        const int64_t kbt = p.k / 64;
        const int kbc = k0 / 64 + (fw >> 3);               // codebook: the word's k-block
        const bool has_dq = KIND == kCode4 && p.q8 != nullptr;
        const float dq_off = has_dq ? __ldg(p.offset) : 0.0f;
        uint32_t mg = 0x43004300u;
        asm volatile("" : "+r"(mg));
        // constants of a block's channels (MinMax scale and zero; codebook
        // absmax, or q8 and s2), loaded two blocks ahead into one of two
        // register sets that the loop below uses in turn (the blocks are
        // processed in pairs, so no register is copied while its load is in
        // flight)
        uint32_t s0[SLOTS], z0[SLOTS], s1[SLOTS], z1[SLOTS];
        auto load_const = [&](int i, uint32_t (&ns)[SLOTS], uint32_t (&nz)[SLOTS]) {
#pragma unroll
            for (int u = 0; u < SLOTS; ++u) {
                const int64_t c = static_cast<int64_t>(blk(i)) * 64 + crow0 + u * cstep;
                if (KIND != kCode4) {
                    ns[u] = c < p.n ? __ldg(p.scale + c * p.ngroups + gcol) : 0u;
                    nz[u] = c < p.n ? __ldg(p.zero + c * p.ngroups + gcol) : 0u;
                } else if (has_dq) {
                    const int64_t e = c * kbt + kbc;
                    ns[u] = c < p.n ? static_cast<uint32_t>(static_cast<int32_t>(__ldg(p.q8 + e))) : 0u;
                    nz[u] = c < p.n ? __float_as_uint(__ldg(p.s2 + (e >> 8))) : 0u;
                } else {
                    ns[u] = c < p.n ? __float_as_uint(__ldg(p.absmax + c * kbt + kbc)) : 0u;
                    nz[u] = 0u;
                }
            }
        };
        if (ncb > 0) load_const(0, s0, z0);
        if (ncb > 1) load_const(1, s1, z1);
        if (lora) {
            // A operand (ring slot 0): K row u = A[u, k0 + feature], features in
            // the tile's pairing order (zero beyond the rank and beyond k)
            const int nunits = p.rank_pad * 16;            // 16-byte units: 8 features of one row
            for (int e = tid; e < nunits; e += 32 * DQW) {
                const int u = e >> 4, fu = e & 15;
                uint32_t wv[4];
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    uint32_t two[2];
#pragma unroll
                    for (int t = 0; t < 2; ++t) {
                        const int pos = fu * 8 + 2 * h + t;
                        const int f = (pos & ~(PG - 1)) + bwd_xperm(KIND, pos & (PG - 1));
                        const int64_t kc = static_cast<int64_t>(k0) + f;
                        two[t] = (u < p.rank && kc < p.k) ? __ldg(p.A + static_cast<int64_t>(u) * p.k + kc) : 0u;
                    }
                    wv[h] = two[0] | (two[1] << 16);
                }
                *reinterpret_cast<uint4*>(sA + bwd_a_offset(u, fu)) = make_uint4(wv[0], wv[1], wv[2], wv[3]);
            }
            // B operand: the tile of bf16(s * U) rows
            stage_scaled_rows(sUop, p.U, t0, min(NT, p.m - t0), NT, p.rank, p.rank_pad, p.s, tid, 32 * DQW);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&afull[0]);
        }
        // block i with its constants cs, cz; false after a timed-out wait
        auto block = [&](int i, const uint32_t (&cs)[SLOTS], const uint32_t (&cz)[SLOTS]) -> bool {
            const int w = i % WS, ia = i + a_off, a = ia % AS;
            if (!mbar_wait(&fullW[w], (i / WS) & 1, s_abort)) return false;
            if (ia >= AS && !mbar_wait(&aempty[a], ((ia / AS) - 1) & 1, s_abort)) return false;
            uint32_t words[SLOTS];
#pragma unroll
            for (int u = 0; u < SLOTS; ++u)
                words[u] = *reinterpret_cast<const uint32_t*>(sW + w * L::kWBytes + (crow0 + u * cstep) * KTB + 4 * fw);
            uint8_t* atile = sA + a * L::kABytes;
#pragma unroll
            for (int u = 0; u < SLOTS; ++u) {
                const int c = crow0 + u * cstep;
                uint32_t o[PG / 2];
                if (KIND == kCode4) {
                    // W_hat = bf16(fp32(codebook[code] * absmax')), rounded once,
                    // in the 4-bit pairing order (codes 1,5 / 0,4 / 3,7 / 2,6)
                    const float a = has_dq ? __fadd_rn(__fmul_rn(__fdiv_rn(static_cast<float>(static_cast<int32_t>(cs[u])),
                                                                           127.0f),
                                                                 __uint_as_float(cz[u])),
                                                       dq_off)
                                           : __uint_as_float(cs[u]);
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        o[q] = pack_bf16x2_rn(__fmul_rn(s_cb[(words[u] >> (4 * q)) & 15u], a),
                                              __fmul_rn(s_cb[(words[u] >> (16 + 4 * q)) & 15u], a));
#pragma unroll
                    for (int h = 0; h < PG / 8; ++h)
                        *reinterpret_cast<uint4*>(atile + bwd_a_offset(c, (PG / 8) * fw + h)) =
                            make_uint4(o[4 * h], o[4 * h + 1], o[4 * h + 2], o[4 * h + 3]);
                    continue;
                }
                const MinMaxConst mc = minmax_const(static_cast<uint16_t>(cs[u]), static_cast<uint16_t>(cz[u]));
                if (BITS == 4)
                    int4_pairs(words[u], mg, o);
                else
                    int2_pairs(words[u], mg, o);
                if (mc.fast) {
#pragma unroll
                    for (int q = 0; q < PG / 2; ++q) o[q] = hsub_hmul_bf16x2(o[q], mc.sub2, mc.mul2);
                } else {
#pragma unroll
                    for (int q = 0; q < PG / 2; ++q)
                        o[q] = minmax_pair_exact((o[q] & 0xFFu), (o[q] >> 16) & 0xFFu, mc);
                }
#pragma unroll
                for (int h = 0; h < PG / 8; ++h)
                    *reinterpret_cast<uint4*>(atile + bwd_a_offset(c, (PG / 8) * fw + h)) =
                        make_uint4(o[4 * h], o[4 * h + 1], o[4 * h + 2], o[4 * h + 3]);
            }
            // the tile was written through the generic proxy; the tensor core reads it through the async one
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&afull[a]);
                mbar_arrive(&emptyW[w]);
            }
            return true;
        };
        for (int i = 0; i < ncb; i += 2) {
            if (!block(i, s0, z0)) break;
            if (i + 2 < ncb) load_const(i + 2, s0, z0);
            if (i + 1 >= ncb) break;
            if (!block(i + 1, s1, z1)) break;
            if (i + 3 < ncb) load_const(i + 3, s1, z1);
        }

        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;                            // TMEM lane quarter of this warp
        const int part = (warp - 2) >> 2;                  // token part
        const int lrow = q * 32 + lane;                    // A-tile row = TMEM lane
        // feature of this lane: the pairing order of its group of PG features
        const int feat = (lrow & ~(PG - 1)) + bwd_xperm(KIND, lrow & (PG - 1));
        const int64_t kcol = k0 + feat;
        const bool col_ok = kcol < p.k;
        const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
        const int mt = min(NT, p.m - t0);
        // (the adapter term is already in the accumulator)
        named_barrier_sync(1, 32 * DQW);
        const bool got = mbar_wait(dfull, 0, s_abort);
        tc_fence_after();
        const bool splitk = p.nsplit > 1;
        constexpr int kPartCols = NT / PARTS >= 16 ? NT / PARTS : 16;
        const int c_begin = part * kPartCols;
        const int c_end = min(NT, c_begin + kPartCols);
        for (int jj = c_begin; jj < c_end; jj += 16) {
            uint32_t raw[16];
            tmem_ld_32x32b_x16(tmem + lane_base + jj, raw);
            tmem_ld_wait();
            if (!col_ok || !got || jj >= mt) continue;
            float acc[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) acc[j] = __uint_as_float(raw[j]);
            if (splitk) {
                float* dst = p.partial + ((static_cast<int64_t>(tl.tile - p.tile0) * p.nsplit + split) * NT + jj) * 128 + lrow;
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    if (jj + j < mt) dst[j * 128] = acc[j];
                continue;
            }
#pragma unroll
            for (int j = 0; j < 16; ++j)
                if (jj + j < mt) p.dX[static_cast<int64_t>(t0 + jj + j) * p.k + kcol] = acc[j];
        }
        if (splitk) {
            __threadfence();
            named_barrier_sync(1, 32 * DQW);
            if (threadIdx.x == 64) {
                const uint32_t tile = tl.tile;
                const uint32_t prev = atomicAdd(p.counters + tile, 1u);
                const int last = (prev == static_cast<uint32_t>(p.nsplit - 1)) ? 1 : 0;
                if (last) p.counters[tile] = 0u;   // left at zero for the next call
                *s_last = last;
            }
            named_barrier_sync(1, 32 * DQW);
            if (*s_last && col_ok && got) {
                __threadfence();
                for (int jj = c_begin; jj < min(c_end, mt); jj += 16) {
                    float acc[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) acc[j] = 0.0f;
                    for (int sp = 0; sp < p.nsplit; ++sp) {
                        const float* src =
                            p.partial + ((static_cast<int64_t>(tl.tile - p.tile0) * p.nsplit + sp) * NT + jj) * 128 + lrow;
                        float part[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) part[j] = (jj + j < mt) ? __ldcg(src + j * 128) : 0.0f;
#pragma unroll
                        for (int j = 0; j < 16; ++j) acc[j] += part[j];
                    }
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        if (jj + j < mt) p.dX[static_cast<int64_t>(t0 + jj + j) * p.k + kcol] = acc[j];
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int NT, int KIND, int XS, int WS, int AS, int MINB, int DQW>
__global__ void __launch_bounds__(fwd_threads(DQW), MINB)
dqgemm_bwd_kernel(const __grid_constant__ CUtensorMap tmDY, const __grid_constant__ CUtensorMap tmW,
                  const BwdParams p) {
    // a one-dimensional grid: nsplit consecutive CTAs per tile, tiles from
    // tile0 on, feature tile fastest
    const int lin = p.tile0 + static_cast<int>(blockIdx.x) / p.nsplit;
    const int split = static_cast<int>(blockIdx.x) % p.nsplit;
    bwd_tile<NT, KIND, XS, WS, AS, DQW>(&tmDY, &tmW, p,
                                        BwdTile{(lin % p.ftiles) * 128, (lin / p.ftiles) * NT, split,
                                                static_cast<uint32_t>(lin)});
}

// A group of backward GEMMs with the same token count in one launch (for
// example the gate and up projections of an MLP): problem i owns CTAs
// cta0[i] .. cta0[i+1]-1, feature tiles fastest, then token tiles, and no
// channel split.  Every CTA runs the kernel above for its problem's weight
// kind (the launch's shared memory fits the largest kind's layout).
constexpr int kBwdMaxGroup = 8;

struct BwdGroupParams {
    CUtensorMap tmDY[kBwdMaxGroup];  // dY of problem i (as for dqgemm_bwd_kernel)
    CUtensorMap tmW[kBwdMaxGroup];   // packed weight of problem i
    BwdParams p[kBwdMaxGroup];
    int kind[kBwdMaxGroup];
    int ftiles[kBwdMaxGroup];        // 128-feature tiles of problem i
    int cta0[kBwdMaxGroup + 1];      // first CTA of problem i; cta0[count] = the grid
    int count;
};

template <int NT, int XS, int WS, int AS, int MINB, int DQW>
__global__ void __launch_bounds__(fwd_threads(DQW), MINB)
dqgemm_bwd_grouped_kernel(const __grid_constant__ BwdGroupParams g) {
    int i = 0;
    for (int j = 1; j < g.count; ++j)
        if (static_cast<int>(blockIdx.x) >= g.cta0[j]) i = j;
    const int local = static_cast<int>(blockIdx.x) - g.cta0[i];
    const BwdTile tl{(local % g.ftiles[i]) * 128, (local / g.ftiles[i]) * NT, 0, static_cast<uint32_t>(local)};
    if (g.kind[i] == kInt4)
        bwd_tile<NT, kInt4, XS, WS, AS, DQW>(&g.tmDY[i], &g.tmW[i], g.p[i], tl);
    else if (g.kind[i] == kInt2)
        bwd_tile<NT, kInt2, XS, WS, AS, DQW>(&g.tmDY[i], &g.tmW[i], g.p[i], tl);
    else
        bwd_tile<NT, kCode4, XS, WS, AS, DQW>(&g.tmDY[i], &g.tmW[i], g.p[i], tl);
}

}  // namespace lbq
