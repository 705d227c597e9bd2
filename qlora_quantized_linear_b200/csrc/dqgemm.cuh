// dqgemm.cuh -- fused dequantize-GEMM on the 5th-generation tensor cores.
//
//   Y[t, c] = sum_k X[t, k] * W_hat[c, k]  (+ s * sum_u T[t, u] B[c, u])
//
// The frozen weight stays packed in HBM (GreenBit.AI article, 模型量化 (1);
// bitsandbytes FSDP-QLoRA guide, 量化数据的存储: codes are unpacked and
// dequantized to the bf16 compute dtype inside the kernel).  One CTA computes
// a tile of 128 output channels x NT tokens:
//
//   warp 0      TMA producer: per k-block of 64, the X tile [NT x 64] bf16
//               (128-byte swizzle, the MMA's B operand) and the packed weight
//               tile [128 rows x 64 codes] into a STAGES-deep smem ring.
//   warp 1      allocates tensor memory; lane 0 issues tcgen05.mma.
//   warps 2..5  dequantize: thread i owns output channel i, which is TMEM
//               lane i.  It unpacks its row's codes from smem, forms bf16
//               W_hat values and stores them with tcgen05.st straight into
//               the MMA's A operand in tensor memory (an ASTAGES-deep ring),
//               so dequantized weights never touch shared memory.  After the
//               last k-block the same threads drain the fp32 accumulator from
//               tensor memory, add the adapter term and write Y.
//
// Decode-sized problems (few tokens) split K across CTAs; each CTA writes an
// fp32 partial tile to the workspace and the last CTA of a tile (found with a
// per-tile counter) sums the partials in split order, so the result does not
// depend on scheduling.  No wait in this kernel spins without a bound.
#pragma once

#include "common.cuh"

namespace lbq {

enum WeightKind : int { kInt4 = 0, kInt2 = 1, kCode4 = 2 };

struct FwdParams {
    int m, n, k;                 // tokens, stored weight rows, input features
    int ngroups;                 // k / group (MinMax)
    const uint16_t* scale;       // [n, ngroups] fp16 (MinMax)
    const uint16_t* zero;        // [n, ngroups] fp16 (MinMax)
    const float* absmax;         // [n * k / 64] (codebook, no double quant)
    const int8_t* q8;            // [n * k / 64] (codebook, double quant)
    const float* s2;             // [ceil(n * k / 64 / 256)]
    const float* offset;         // [1]
    const float* codebook;       // [16]
    int rank;                    // adapter rank, 0 = none
    int rank_pad;                // rank rounded up to 16 (row stride of the staged T tile)
    float s;                     // adapter scale
    const float* T;              // [m, rank] fp32
    const uint16_t* B;           // [n_out, rank] bf16, indexed by output column
    float* Y;                    // output, Y[t * ldy + out_col]
    int64_t ldy;
    const int32_t* perm;         // stored row -> output column (NULL = identity)
    int kb_per_split;            // k-blocks of 64 per split
    int nsplit;
    float* partial;              // [nsplit, m, n] fp32 (nsplit > 1)
    uint32_t* counters;          // [tiles] (nsplit > 1), zero between calls
};

template <int KIND>
struct WeightTile {
    static constexpr int kRowBytes = (KIND == kInt2) ? 16 : 32;  // packed bytes per row per k-block
};

// Shared-memory layout of one CTA: a ring of STAGES (activation tile, packed
// weight tile) pairs, the mbarriers, and the adapter T tile [NT, rank_pad].
template <int NT, int STAGES, int ASTAGES, int WTILE>
struct GemmSmem {
    static constexpr int kXBytes = NT * 128;   // NT rows x 64 bf16
    static constexpr int kWBytes = WTILE;      // packed weight tile
    static constexpr size_t kX = 0;
    static constexpr size_t kW = kX + size_t(STAGES) * kXBytes;
    static constexpr size_t kBar = (kW + size_t(STAGES) * kWBytes + 7) / 8 * 8;
    static constexpr int kNumBars = 2 * STAGES + 2 * ASTAGES + 1;
    static constexpr size_t kMisc = kBar + kNumBars * 8;
    static constexpr size_t kTab = (kMisc + 128 + 15) / 16 * 16;   // per-stage dequant tables (backward)
    static constexpr size_t kTabBytes = 64 * 2 * 16;
    static constexpr size_t kLoraT = kTab + size_t(STAGES) * kTabBytes;
    static size_t total(int rank_pad) { return kLoraT + size_t(NT) * rank_pad * 4 + 1024; }
};

__host__ __device__ constexpr uint32_t tmem_cols_for(int ncols) {
    return ncols <= 32 ? 32 : ncols <= 64 ? 64 : ncols <= 128 ? 128 : ncols <= 256 ? 256 : 512;
}

// Four bf16x2 registers (first code in the low half) from one word of packed
// 4-bit codes; byte j holds codes 2j (high nibble) and 2j+1 (low nibble).
// Each half is the bf16 number 128 + code.
__device__ __forceinline__ void unpack_int4_word(uint32_t w, uint32_t (&o)[4]) {
    const uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;
    const uint32_t lo = w & 0x0F0F0F0Fu;
    const uint32_t m = 0x43434343u;
    const uint32_t p01 = __byte_perm(hi, lo, 0x5140);  // h0 l0 h1 l1
    const uint32_t p23 = __byte_perm(hi, lo, 0x7362);  // h2 l2 h3 l3
    o[0] = __byte_perm(p01, m, 0x4140);
    o[1] = __byte_perm(p01, m, 0x4342);
    o[2] = __byte_perm(p23, m, 0x4140);
    o[3] = __byte_perm(p23, m, 0x4342);
}

// Eight bf16x2 registers from one word of packed 2-bit codes; byte j holds
// codes 4j..4j+3 from the top bits down.
__device__ __forceinline__ void unpack_int2_word(uint32_t w, uint32_t (&o)[8]) {
    const uint32_t c0 = (w >> 6) & 0x03030303u, c1 = (w >> 4) & 0x03030303u;
    const uint32_t c2 = (w >> 2) & 0x03030303u, c3 = w & 0x03030303u;
    const uint32_t m = 0x43434343u;
    const uint32_t a01 = __byte_perm(c0, c1, 0x5140), a23 = __byte_perm(c0, c1, 0x7362);
    const uint32_t b01 = __byte_perm(c2, c3, 0x5140), b23 = __byte_perm(c2, c3, 0x7362);
    o[0] = __byte_perm(a01, m, 0x4140);  // byte 0: codes 0, 1
    o[1] = __byte_perm(b01, m, 0x4140);  // byte 0: codes 2, 3
    o[2] = __byte_perm(a01, m, 0x4342);  // byte 1
    o[3] = __byte_perm(b01, m, 0x4342);
    o[4] = __byte_perm(a23, m, 0x4140);  // byte 2
    o[5] = __byte_perm(b23, m, 0x4140);
    o[6] = __byte_perm(a23, m, 0x4342);  // byte 3
    o[7] = __byte_perm(b23, m, 0x4342);
}

__device__ __forceinline__ uint32_t hsub_hmul_bf16x2(uint32_t v, uint32_t sub, uint32_t mul) {
    __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&v);
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&sub);
    const __nv_bfloat162 c = *reinterpret_cast<const __nv_bfloat162*>(&mul);
    a = __hmul2(__hsub2(a, b), c);
    return *reinterpret_cast<uint32_t*>(&a);
}

// Per-row, per-group dequantization constants of the MinMax format.
struct MinMaxConst {
    uint32_t sub2;   // bf16x2 (128 + zero) in both halves
    uint32_t mul2;   // bf16x2 scale (rounded to bf16) in both halves
    float sf, zf;    // exact scale and zero (fp32)
    bool fast;       // |zero| <= 128: 128 + zero and code - zero are exact in bf16
};

__device__ __forceinline__ MinMaxConst minmax_const(uint16_t s16, uint16_t z16) {
    MinMaxConst c;
    c.sf = f16_bits_to_f32(s16);
    c.zf = f16_bits_to_f32(z16);
    c.fast = fabsf(c.zf) <= 128.0f;
    c.sub2 = pack_bf16x2_rn(128.0f + c.zf, 128.0f + c.zf);
    c.mul2 = pack_bf16x2_rn(c.sf, c.sf);
    return c;
}

// Exact path: bf16(fp32((code - zero) * scale)) for a pair of codes.
__device__ __forceinline__ uint32_t minmax_pair_exact(uint32_t q0, uint32_t q1, const MinMaxConst& c) {
    const float w0 = __fmul_rn(__fsub_rn(static_cast<float>(q0), c.zf), c.sf);
    const float w1 = __fmul_rn(__fsub_rn(static_cast<float>(q1), c.zf), c.sf);
    return pack_bf16x2_rn(w0, w1);
}

// Dequantize this thread's row of one k-block (64 codes) into 32 bf16x2 words.
template <int KIND>
__device__ __forceinline__ void dequant_row_kblock(const uint8_t* wrow_smem, int row, int kb, int64_t grow,
                                                   const FwdParams& p, const float* s_cb, uint32_t (&out)[32]) {
    if (KIND == kInt4) {
        // 32 bytes, stored by TMA with the 32-byte swizzle: 16-byte chunk c of
        // row r sits at chunk c ^ ((r >> 2) & 1).
        const int sw = (row >> 2) & 1;
        const uint4 c0 = *reinterpret_cast<const uint4*>(wrow_smem + 16 * (0 ^ sw));
        const uint4 c1 = *reinterpret_cast<const uint4*>(wrow_smem + 16 * (1 ^ sw));
        const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        const int g = (kb * 64) / 128;
        const MinMaxConst c = minmax_const(__ldg(p.scale + grow * p.ngroups + g), __ldg(p.zero + grow * p.ngroups + g));
        if (c.fast) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                uint32_t o[4];
                unpack_int4_word(w[i], o);
#pragma unroll
                for (int j = 0; j < 4; ++j) out[4 * i + j] = hsub_hmul_bf16x2(o[j], c.sub2, c.mul2);
            }
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    out[4 * i + j] = minmax_pair_exact((w[i] >> (8 * j + 4)) & 15u, (w[i] >> (8 * j)) & 15u, c);
        }
    } else if (KIND == kInt2) {
        const uint4 c0 = *reinterpret_cast<const uint4*>(wrow_smem);
        const uint32_t w[4] = {c0.x, c0.y, c0.z, c0.w};
        const int g = kb;  // group 64 == k-block
        const MinMaxConst c = minmax_const(__ldg(p.scale + grow * p.ngroups + g), __ldg(p.zero + grow * p.ngroups + g));
        if (c.fast) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                uint32_t o[8];
                unpack_int2_word(w[i], o);
#pragma unroll
                for (int j = 0; j < 8; ++j) out[8 * i + j] = hsub_hmul_bf16x2(o[j], c.sub2, c.mul2);
            }
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j)
#pragma unroll
                    for (int h = 0; h < 2; ++h)
                        out[8 * i + 2 * j + h] = minmax_pair_exact((w[i] >> (8 * j + 6 - 4 * h)) & 3u,
                                                                   (w[i] >> (8 * j + 4 - 4 * h)) & 3u, c);
        }
    } else {
        // codebook: W_hat = bf16(fp32(codebook[code] * absmax)), absmax per 64
        const int sw = (row >> 2) & 1;
        const uint4 c0 = *reinterpret_cast<const uint4*>(wrow_smem + 16 * (0 ^ sw));
        const uint4 c1 = *reinterpret_cast<const uint4*>(wrow_smem + 16 * (1 ^ sw));
        const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
        const int64_t b = grow * (p.k / 64) + kb;
        float a;
        if (p.q8 != nullptr) {
            a = __fadd_rn(__fmul_rn(__fdiv_rn(static_cast<float>(__ldg(p.q8 + b)), 127.0f), __ldg(p.s2 + (b >> 8))),
                          __ldg(p.offset));
        } else {
            a = __ldg(p.absmax + b);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j)
                out[4 * i + j] = pack_bf16x2_rn(__fmul_rn(s_cb[(w[i] >> (8 * j + 4)) & 15u], a),
                                                __fmul_rn(s_cb[(w[i] >> (8 * j)) & 15u], a));
    }
}

// acc[j] += s * sum_u Trow_j[u] * b[u] for 16 consecutive tokens j, where
// Trow_j = sT + j * rp (fp32, zero-padded to rp) and b[u] = brow[u * bstride]
// (bf16): B[out_col, :] in the forward pass, A[:, k] in the backward pass.
__device__ __forceinline__ void lora_add16(float (&acc)[16], const float* sT, int rp, int rank,
                                           const uint16_t* brow, float s, int64_t bstride = 1) {
    float d[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) d[j] = 0.0f;
    for (int u0 = 0; u0 < rp; u0 += 16) {
        float b[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) b[u] = (u0 + u < rank) ? bf16_bits_to_f32(__ldg(brow + (u0 + u) * bstride)) : 0.0f;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const float4* t4 = reinterpret_cast<const float4*>(sT + j * rp + u0);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const float4 t = t4[v];
                d[j] = fmaf(t.x, b[4 * v], d[j]);
                d[j] = fmaf(t.y, b[4 * v + 1], d[j]);
                d[j] = fmaf(t.z, b[4 * v + 2], d[j]);
                d[j] = fmaf(t.w, b[4 * v + 3], d[j]);
            }
        }
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) acc[j] = fmaf(s, d[j], acc[j]);
}

template <int NT, int KIND, int STAGES, int ASTAGES>
__global__ void __launch_bounds__(192, 2)
dqgemm_fwd_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                  const FwdParams p) {
    constexpr int WB = WeightTile<KIND>::kRowBytes;
    using L = GemmSmem<NT, STAGES, ASTAGES, 128 * WB>;
    constexpr uint32_t kTxBytes = L::kXBytes + 128 * WB;
    constexpr int kACols = 32;                         // one k-block of 64 bf16 = 32 columns
    constexpr int kDCol = 0;                           // fp32 accumulator: NT columns
    constexpr int kACol0 = (NT + 31) / 32 * 32;        // A ring after the accumulator
    constexpr uint32_t kTmemCols = tmem_cols_for(kACol0 + kACols * ASTAGES);
    constexpr uint32_t kIdesc = idesc_bf16_f32(128, NT);

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
    float* s_cb = reinterpret_cast<float*>(smem + L::kMisc + 64);  // 16 floats
    float* sT = reinterpret_cast<float*>(smem + L::kLoraT);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * 128;
    const int t0 = blockIdx.y * NT;
    const int split = blockIdx.z;
    const int kb_total = p.k / 64;
    const int kb0 = split * p.kb_per_split;
    const int nkb = min(p.kb_per_split, kb_total - kb0);

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
    if (KIND == kCode4 && threadIdx.x < 16) s_cb[threadIdx.x] = p.codebook[threadIdx.x];
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmX);
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
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            int issued = 0;
            for (int i = 0; i < nkb; ++i) {
                const int s = i % STAGES;
                if (i >= STAGES && !mbar_wait(&empty[s], ((i / STAGES) - 1) & 1, s_abort)) break;
                mbar_arrive_expect_tx(&full[s], kTxBytes);
                const int kb = kb0 + i;
                tma_load_2d(sX + s * L::kXBytes, &tmX, &full[s], kb * 64, t0);
                tma_load_2d(sW + s * L::kWBytes, &tmW, &full[s], kb * WB, n0);
                issued = i + 1;
            }
            // never leave with a copy in flight (matters only after an abort)
            for (int i = max(0, issued - STAGES); i < issued; ++i) mbar_wait_drain(&full[i % STAGES], (i / STAGES) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            bool ok = true;
            for (int i = 0; i < nkb && ok; ++i) {
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
            mma_commit(dfull);  // also completes when nothing was issued
            mbar_wait_drain(dfull, 0);  // MMAs done before tensor memory is freed
        }
    } else {
        // ------------------------------------------------------------ dequantize
        const int q = warp & 3;            // TMEM lane quarter of this warp
        const int row = q * 32 + lane;     // output channel within the tile
        const int64_t grow = n0 + row;     // stored weight row
        const bool row_ok = grow < p.n;
        const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
        for (int i = 0; i < nkb; ++i) {
            const int s = i % STAGES, a = i % ASTAGES;
            if (!mbar_wait(&full[s], (i / STAGES) & 1, s_abort)) break;
            if (i >= ASTAGES && !mbar_wait(&aempty[a], ((i / ASTAGES) - 1) & 1, s_abort)) break;
            tc_fence_after();
            uint32_t vals[32];
            if (row_ok) {
                dequant_row_kblock<KIND>(sW + s * L::kWBytes + row * WB, row, kb0 + i, grow, p, s_cb, vals);
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j) vals[j] = 0u;
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
        const int mt = min(NT, p.m - t0);  // tokens in this tile
        const bool lora = p.rank > 0;
        // stage T[t0 : t0 + mt, :rank] (fp32) in smem for the adapter term
        if (lora) {
            const int tid = threadIdx.x - 64;
            for (int e = tid; e < NT * p.rank_pad; e += 128) {
                const int tt = e / p.rank_pad, u = e - tt * p.rank_pad;
                sT[e] = (tt < mt && u < p.rank) ? p.T[static_cast<int64_t>(t0 + tt) * p.rank + u] : 0.0f;
            }
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
        const bool got = mbar_wait(dfull, 0, s_abort);
        tc_fence_after();
        const int out_col = row_ok ? (p.perm ? p.perm[grow] : static_cast<int>(grow)) : 0;
        const int rp = p.rank_pad;
        const bool splitk = p.nsplit > 1;
        for (int jj = 0; jj < NT; jj += 16) {
            uint32_t raw[16];
            tmem_ld_32x32b_x16(tmem + lane_base + kDCol + jj, raw);
            tmem_ld_wait();
            if (!row_ok || !got || jj >= mt) continue;
            float acc[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) acc[j] = __uint_as_float(raw[j]);
            if (splitk) {
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    if (jj + j < mt) p.partial[(static_cast<int64_t>(split) * p.m + t0 + jj + j) * p.n + grow] = acc[j];
                continue;
            }
            if (lora) lora_add16(acc, sT + jj * rp, rp, p.rank, p.B + static_cast<int64_t>(out_col) * p.rank, p.s);
#pragma unroll
            for (int j = 0; j < 16; ++j)
                if (jj + j < mt) p.Y[static_cast<int64_t>(t0 + jj + j) * p.ldy + out_col] = acc[j];
        }
        if (splitk) {
            // the last CTA of this output tile sums the partials in split order
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
            if (*s_last && row_ok && got) {
                __threadfence();
                for (int jj = 0; jj < mt; jj += 16) {
                    float acc[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        acc[j] = 0.0f;
                        if (jj + j < mt)
                            for (int sp = 0; sp < p.nsplit; ++sp)
                                acc[j] += __ldcg(p.partial + (static_cast<int64_t>(sp) * p.m + t0 + jj + j) * p.n + grow);
                    }
                    if (lora) lora_add16(acc, sT + jj * rp, rp, p.rank, p.B + static_cast<int64_t>(out_col) * p.rank, p.s);
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        if (jj + j < mt) p.Y[static_cast<int64_t>(t0 + jj + j) * p.ldy + out_col] = acc[j];
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
