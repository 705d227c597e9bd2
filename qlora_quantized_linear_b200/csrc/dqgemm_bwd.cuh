// dqgemm_bwd.cuh -- input gradient through the frozen quantized weight on the
// 5th-generation tensor cores (QLoRA explainer, QLoRA技术原理: gradients flow
// through the frozen 4-bit weight into the adapters):
//
//   dX[t, k] = sum_c dY[t, c] * W_hat[c, k]  (+ s * sum_u U[t, u] A[u, k])
//
// The weight is read in its stored [n, k] packed layout -- no transposed copy
// exists.  One CTA computes a tile of 128 input features x NT tokens: thread i
// of the dequantize warps owns input feature k0 + i (TMEM lane i) and, for each
// block of 64 output channels c, gathers its column of codes from the staged
// packed tile, so the MMA's A operand in tensor memory is W_hat^T with the
// reduction over c along the columns.  dY tiles [NT x 64 c] arrive by TMA as
// the B operand.  Per-channel scale/zero constants of each block are built
// once per block into a shared-memory table.  Roles, rings, bounded waits and
// the split-K reduction mirror the forward kernel.
#pragma once

#include "dqgemm.cuh"

namespace lbq {

struct BwdParams {
    int m, n, k;                 // tokens, weight rows (output channels), input features
    int bits, ngroups;           // MinMax bit width, k / group
    const uint16_t* scale;       // [n, ngroups]
    const uint16_t* zero;        // [n, ngroups]
    int rank, rank_pad;
    float s;
    const float* U;              // [m, rank] fp32
    const uint16_t* A;           // [rank, k] bf16
    float* dX;                   // [m, k]
    int cb_per_split;            // blocks of 64 output channels per split
    int nsplit;
    float* partial;              // [nsplit, m, k]
    uint32_t* counters;
};

// Two table buffers of 2048 bytes: G*32 PairConst + G*64 float2 each.
constexpr int kBwdTabBytes = 4096;

// Dequantization constants of one channel pair for one group (bf16x2 fast
// path) and of single channels (fp32 exact path).
struct PairConst {
    uint32_t sub2, mul2;
    uint32_t fast, pad;
};

template <int NT, int BITS, int STAGES, int ASTAGES>
__global__ void __launch_bounds__(192, 2)
dqgemm_bwd_kernel(const __grid_constant__ CUtensorMap tmDY, const __grid_constant__ CUtensorMap tmW,
                  const BwdParams p) {
    constexpr int KTB = 128 * BITS / 8;       // packed bytes of one row across the 128-feature tile
    constexpr int G = (BITS == 4) ? 1 : 2;    // groups covered by the 128-feature tile
    using L = GemmSmem<NT, STAGES, ASTAGES, 64 * KTB, kBwdTabBytes>;
    constexpr uint32_t kTxBytes = L::kXBytes + 64 * KTB;
    constexpr int kACols = 32;
    constexpr int kDCol = 0;
    constexpr int kACol0 = (NT + 31) / 32 * 32;
    constexpr uint32_t kTmemCols = tmem_cols_for(kACol0 + kACols * ASTAGES);
    constexpr uint32_t kIdesc = idesc_bf16_f32(128, NT);
    constexpr int kTabBuf = kBwdTabBytes / 2;  // one table buffer: G*32 PairConst + G*64 float2

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sX = smem + L::kX;
    uint8_t* sW = smem + L::kW;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
    uint64_t* full = bars;
    uint64_t* empty = bars + STAGES;
    uint64_t* afull = bars + 2 * STAGES;
    uint64_t* aempty = afull + ASTAGES;
    uint64_t* dfull = aempty + ASTAGES;
    uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + L::kMisc);
    volatile int* s_abort = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);
    int* s_last = reinterpret_cast<int*>(smem + L::kMisc + 8);
    // two table buffers: [G][32 pairs] PairConst, then [G][64 channels] float2 (sf, zf)
    uint8_t* s_tab = smem + L::kTab;
    float* sT = reinterpret_cast<float*>(smem + L::kLoraT);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int k0 = blockIdx.x * 128;
    const int t0 = blockIdx.y * NT;
    const int split = blockIdx.z;
    const int cb_total = (p.n + 63) / 64;
    const int cb0 = split * p.cb_per_split;
    const int ncb = min(p.cb_per_split, cb_total - cb0);

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1 + 4);
        }
        for (int i = 0; i < ASTAGES; ++i) {
            mbar_init(&afull[i], 4);
            mbar_init(&aempty[i], 1);
        }
        mbar_init(dfull, 1);
        *s_abort = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmDY);
        tma_prefetch_desc(&tmW);
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
        if (lane == 0) {
            int issued = 0;
            for (int i = 0; i < ncb; ++i) {
                const int s = i % STAGES;
                if (i >= STAGES && !mbar_wait(&empty[s], ((i / STAGES) - 1) & 1, s_abort)) break;
                mbar_arrive_expect_tx(&full[s], kTxBytes);
                const int c0 = (cb0 + i) * 64;
                tma_load_2d(sX + s * L::kXBytes, &tmDY, &full[s], c0, t0);
                tma_load_2d(sW + s * L::kWBytes, &tmW, &full[s], k0 * BITS / 8, c0);
                issued = i + 1;
            }
            for (int i = max(0, issued - STAGES); i < issued; ++i) mbar_wait_drain(&full[i % STAGES], (i / STAGES) & 1);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            bool ok = true;
            for (int i = 0; i < ncb && ok; ++i) {
                const int s = i % STAGES, a = i % ASTAGES;
                ok = mbar_wait(&full[s], (i / STAGES) & 1, s_abort) &&
                     mbar_wait(&afull[a], (i / ASTAGES) & 1, s_abort);
                if (!ok) break;
                tc_fence_after();
                const uint64_t bdesc = smem_desc_k_sw128(smem_u32(sX + s * L::kXBytes));
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    mma_ts(tmem + kDCol, tmem + kACol0 + a * kACols + 8 * j, bdesc + static_cast<uint64_t>(2 * j), kIdesc,
                           (i > 0 || j > 0) ? 1u : 0u);
                mma_commit(&empty[s]);
                mma_commit(&aempty[a]);
            }
            mma_commit(dfull);
            mbar_wait_drain(dfull, 0);
        }
    } else {
        const int q = warp & 3;
        const int r = q * 32 + lane;            // feature within the tile = TMEM lane
        const int64_t kcol = k0 + r;
        const bool col_ok = kcol < p.k;
        const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
        const int tid = threadIdx.x - 64;       // 0..127
        const int bytecol = (BITS == 4) ? (r >> 1) : (r >> 2);
        const int sh = (BITS == 4) ? ((r & 1) ? 0 : 4) : (6 - 2 * (r & 3));
        const uint32_t msk = (BITS == 4) ? 0x000F000Fu : 0x00030003u;
        const int gi = (G == 1) ? 0 : (r >> 6);
        bool dead = false;  // after an abort: keep meeting the named barriers, skip the work
        for (int i = 0; i < ncb; ++i) {
            const int s = i % STAGES, a = i % ASTAGES;
            const int c0 = (cb0 + i) * 64;
            // --- constants of this block's 64 channels, built by the 128 threads
            PairConst* tabp = reinterpret_cast<PairConst*>(s_tab + (i & 1) * kTabBuf);
            float2* tabs = reinterpret_cast<float2*>(s_tab + (i & 1) * kTabBuf + G * 32 * sizeof(PairConst));
            if (tid < 64 * G) {
                const int cl = tid & 63, g = tid >> 6;
                const int64_t c = c0 + cl;
                float sf = 0.0f, zf = 0.0f;
                if (c < p.n) {
                    const int gg = (k0 / (BITS == 4 ? 128 : 64)) + g;
                    sf = f16_bits_to_f32(__ldg(p.scale + c * p.ngroups + gg));
                    zf = f16_bits_to_f32(__ldg(p.zero + c * p.ngroups + gg));
                }
                tabs[g * 64 + cl] = make_float2(sf, zf);
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (tid < 32 * G) {
                const int pp = tid & 31, g = tid >> 5;
                const float2 e0 = tabs[g * 64 + 2 * pp], e1 = tabs[g * 64 + 2 * pp + 1];
                PairConst pc;
                pc.sub2 = pack_bf16x2_rn(128.0f + e0.y, 128.0f + e1.y);
                pc.mul2 = pack_bf16x2_rn(e0.x, e1.x);
                pc.fast = (fabsf(e0.y) <= 128.0f && fabsf(e1.y) <= 128.0f) ? 1u : 0u;
                pc.pad = 0;
                tabp[g * 32 + pp] = pc;
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
            dead = dead || !mbar_wait(&full[s], (i / STAGES) & 1, s_abort);
            dead = dead || (i >= ASTAGES && !mbar_wait(&aempty[a], ((i / ASTAGES) - 1) & 1, s_abort));
            if (dead) continue;
            tc_fence_after();
            uint32_t vals[32];
            const uint8_t* wt = sW + s * L::kWBytes + bytecol;
#pragma unroll
            for (int pp = 0; pp < 32; ++pp) {
                const uint32_t b0 = wt[(2 * pp) * KTB];
                const uint32_t b1 = wt[(2 * pp + 1) * KTB];
                const uint32_t t = __byte_perm(b0, b1, 0x5410);
                const PairConst pc = tabp[gi * 32 + pp];
                if (pc.fast) {
                    const uint32_t v = ((t >> sh) & msk) | 0x43004300u;
                    vals[pp] = hsub_hmul_bf16x2(v, pc.sub2, pc.mul2);
                } else {
                    const float2 e0 = tabs[gi * 64 + 2 * pp], e1 = tabs[gi * 64 + 2 * pp + 1];
                    const float w0 = __fmul_rn(__fsub_rn(static_cast<float>((t >> sh) & (msk & 0xFFFFu)), e0.y), e0.x);
                    const float w1 = __fmul_rn(__fsub_rn(static_cast<float>((t >> (sh + 16)) & (msk & 0xFFFFu)), e1.y), e1.x);
                    vals[pp] = pack_bf16x2_rn(w0, w1);
                }
            }
            tmem_st_32x32b_x32(tmem + lane_base + kACol0 + a * kACols, vals);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&afull[a]);
                mbar_arrive(&empty[s]);
            }
        }

        // ------------------------------------------------------------ epilogue
        const int mt = min(NT, p.m - t0);
        const bool lora = p.rank > 0;
        if (lora) {
            for (int e = tid; e < NT * p.rank_pad; e += 128) {
                const int tt = e / p.rank_pad, u = e - tt * p.rank_pad;
                sT[e] = (tt < mt && u < p.rank) ? p.U[static_cast<int64_t>(t0 + tt) * p.rank + u] : 0.0f;
            }
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        const bool got = mbar_wait(dfull, 0, s_abort);
        tc_fence_after();
        const int rp = p.rank_pad;
        const bool splitk = p.nsplit > 1;
        for (int jj = 0; jj < NT; jj += 16) {
            uint32_t raw[16];
            tmem_ld_32x32b_x16(tmem + lane_base + kDCol + jj, raw);
            tmem_ld_wait();
            if (!col_ok || !got || jj >= mt) continue;
            float acc[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) acc[j] = __uint_as_float(raw[j]);
            if (splitk) {
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    if (jj + j < mt) p.partial[(static_cast<int64_t>(split) * p.m + t0 + jj + j) * p.k + kcol] = acc[j];
                continue;
            }
            if (lora) lora_add16(acc, sT + jj * rp, rp, p.rank, p.A + kcol, p.s, p.k);
#pragma unroll
            for (int j = 0; j < 16; ++j)
                if (jj + j < mt) p.dX[static_cast<int64_t>(t0 + jj + j) * p.k + kcol] = acc[j];
        }
        if (splitk) {
            __threadfence();
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (threadIdx.x == 64) {
                const uint32_t tile = blockIdx.y * gridDim.x + blockIdx.x;
                const uint32_t prev = atomicAdd(p.counters + tile, 1u);
                const int last = (prev == static_cast<uint32_t>(p.nsplit - 1)) ? 1 : 0;
                if (last) p.counters[tile] = 0u;
                *s_last = last;
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (*s_last && col_ok && got) {
                __threadfence();
                for (int jj = 0; jj < mt; jj += 16) {
                    float acc[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        acc[j] = 0.0f;
                        if (jj + j < mt)
                            for (int sp = 0; sp < p.nsplit; ++sp)
                                acc[j] += __ldcg(p.partial + (static_cast<int64_t>(sp) * p.m + t0 + jj + j) * p.k + kcol);
                    }
                    if (lora) lora_add16(acc, sT + jj * rp, rp, p.rank, p.A + kcol, p.s, p.k);
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

}  // namespace lbq
