// dqgemm.cuh -- fused dequantize-GEMM on the 5th-generation tensor cores.
//
//   Y[t, c] = sum_k X[t, k] * W_hat[c, k]  (+ s * sum_u T[t, u] B[c, u])
//
// The frozen weight stays packed in HBM (GreenBit.AI article, 模型量化 (1);
// bitsandbytes FSDP-QLoRA guide, 量化数据的存储: codes are unpacked and
// dequantized to the bf16 compute dtype inside the kernel).  One CTA computes
// a tile of 128 output channels x NT tokens:
//
//   warp 0      TMA producer: X tiles [NT x 64] bf16 (128-byte swizzle, the
//               MMA's B operand), several k-blocks per 3-D box, into one ring;
//               the packed weights in chunks of 128 rows x 128 bytes (256
//               INT4 or 512 INT2 codes per row, 128-byte swizzle) into a
//               second ring -- wide boxes keep the TMA engine efficient.
//   warp 1      allocates tensor memory; lane 0 issues tcgen05.mma.
//   warps 2..   dequantize (16 warps for the 256-token tile, else 8): output
//               channel i is TMEM lane i; the warps of a lane quarter each
//               take one part (a quarter or a half) of a k-block.  A thread
//               unpacks its row's codes from smem, forms bf16 W_hat values and
//               stores them with tcgen05.st straight into the MMA's A operand
//               in tensor memory (an ASTAGES-deep ring), so dequantized
//               weights never touch shared memory.  Per-row scale/zero are
//               loaded one k-block ahead.  After the last k-block the same
//               threads drain the fp32 accumulator from tensor memory, add
//               the adapter term and write Y.
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
    int nsplit;                  // splits of every tile of this launch
    int tile0;                   // first tile of this launch (tiles numbered row tile fastest)
    int rtiles;                  // 128-row tiles of the GEMM
    float* partial;              // [tile - tile0][nsplit][NT tokens][128 rows] fp32 (nsplit > 1)
    uint32_t* counters;          // [tiles] (nsplit > 1), zero between calls
};

template <int KIND>
struct WeightTile {
    static constexpr int kRowBytes = (KIND == kInt2) ? 16 : 32;  // packed bytes per row per k-block
    // The forward kernel loads weights in chunks of 128 bytes per row (a
    // 128-row x 128-byte box, 128-byte swizzle): kSub k-blocks per chunk.
    static constexpr int kSub = 128 / kRowBytes;
};

// Shared-memory layout of the forward kernel: a ring of XS activation slots
// (XB k-blocks of NT x 64 bf16 each, fetched by one 3-D TMA box), a ring of
// WS packed-weight chunks (128 rows x 128 B), the mbarriers and, with an
// adapter, the MMA operand tile of s*T [NT tokens x 64 rank] (bf16, K-major,
// 128-byte swizzle).  Few, large TMA boxes: each box costs the TMA engine a
// fixed issue-to-completion slot, so small boxes waste its throughput.
template <int NT, int XS, int XB, int WS, int AS>
struct FwdSmem {
    static constexpr int kXTile = NT * 128;              // one k-block of X
    static constexpr int kXBytes = XB * kXTile;          // one X slot
    static constexpr int kWBytes = 128 * 128;
    static constexpr size_t kX = 0;
    static constexpr size_t kW = kX + size_t(XS) * kXBytes;
    static constexpr size_t kBar = kW + size_t(WS) * kWBytes;
    static constexpr int kNumBars = 2 * XS + 2 * WS + 2 * AS + 1;
    static constexpr size_t kMisc = kBar + kNumBars * 8;
    static constexpr size_t kLoraT = (kMisc + 128 + 1023) / 1024 * 1024;
    static size_t total(int rank) { return kLoraT + (rank > 0 ? size_t(NT) * 128 : 0) + 1024; }
};

// Shared-memory layout of one CTA: a ring of STAGES (activation tile, packed
// weight tile) pairs, the mbarriers, and the adapter T tile [NT, rank_pad].
template <int NT, int STAGES, int ASTAGES, int WTILE, int TABBYTES = 0>
struct GemmSmem {
    static constexpr int kXBytes = NT * 128;   // NT rows x 64 bf16
    static constexpr int kWBytes = WTILE;      // packed weight tile
    static constexpr size_t kX = 0;
    static constexpr size_t kW = kX + size_t(STAGES) * kXBytes;
    static constexpr size_t kBar = (kW + size_t(STAGES) * kWBytes + 7) / 8 * 8;
    static constexpr int kNumBars = 2 * STAGES + 2 * ASTAGES + 1;
    static constexpr size_t kMisc = kBar + kNumBars * 8;
    static constexpr size_t kTab = (kMisc + 128 + 15) / 16 * 16;   // dequant tables (backward only)
    static constexpr size_t kLoraT = kTab + size_t(TABBYTES);
    static size_t total(int rank_pad) { return kLoraT + size_t(NT) * rank_pad * 4 + 1024; }
};

// bar.sync on barrier `id` for `count` threads (a multiple of 32).
__device__ __forceinline__ void named_barrier_sync(int id, int count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

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

__device__ __forceinline__ uint32_t hsub_bf16x2(uint32_t v, uint32_t sub) {
    __nv_bfloat162 a = *reinterpret_cast<__nv_bfloat162*>(&v);
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(&sub);
    a = __hsub2(a, b);
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

// Raw per-(row, k-block) constants, loaded one k-block ahead of their use so
// that the load latency hides behind the previous block's dequantization.
struct PreConst {
    uint32_t a, b;   // MinMax: scale bits, zero bits; codebook: absmax bits or (q8, s2 bits)
};

template <int KIND>
__device__ __forceinline__ PreConst preload_const(const FwdParams& p, int64_t grow, int kb, bool ok) {
    PreConst c{0u, 0u};
    if (!ok) return c;
    if (KIND != kCode4) {
        const int g = (KIND == kInt4) ? (kb >> 1) : kb;
        c.a = __ldg(p.scale + grow * p.ngroups + g);
        c.b = __ldg(p.zero + grow * p.ngroups + g);
    } else {
        const int64_t b = grow * (p.k / 64) + kb;
        if (p.q8 != nullptr) {
            c.a = static_cast<uint32_t>(static_cast<int32_t>(__ldg(p.q8 + b)));
            c.b = __float_as_uint(__ldg(p.s2 + (b >> 8)));
        } else {
            c.a = __float_as_uint(__ldg(p.absmax + b));
        }
    }
    return c;
}

// Dequantize part of this thread's row of one k-block (2 NV codes) into NV
// bf16x2 words (first code of each pair in the low half).  `wrow` is the row's
// 128-byte line of the weight chunk, stored by TMA with the 128-byte swizzle
// (16-byte unit u of row r sits at unit u ^ (r & 7)); `byte0` is the offset of
// the part's codes within the line.
template <int KIND, int NV>
__device__ __forceinline__ void dequant_part_kblock(const uint8_t* wrow, int row, int byte0, PreConst pc,
                                                    const MinMaxConst& c, float dq_offset, bool has_dq,
                                                    const float* s_cb, uint32_t (&out)[NV]) {
    constexpr int NW = (KIND == kInt2) ? NV / 8 : NV / 4;   // 32-bit words of codes
    const uint8_t* src = wrow + 16 * ((byte0 >> 4) ^ (row & 7)) + (byte0 & 15);
    uint32_t w[NW];
    if (NW == 4) {
        const uint4 c = *reinterpret_cast<const uint4*>(src);
        w[0] = c.x;
        w[1 % NW] = c.y;
        w[2 % NW] = c.z;
        w[3 % NW] = c.w;
    } else if (NW == 2) {
        const uint2 c = *reinterpret_cast<const uint2*>(src);
        w[0] = c.x;
        w[1 % NW] = c.y;
    } else {
        w[0] = *reinterpret_cast<const uint32_t*>(src);
    }
    if (KIND == kInt4) {
        if (c.fast) {
#pragma unroll
            for (int i = 0; i < NW; ++i) {
                uint32_t o[4];
                unpack_int4_word(w[i], o);
#pragma unroll
                for (int j = 0; j < 4; ++j) out[4 * i + j] = hsub_hmul_bf16x2(o[j], c.sub2, c.mul2);
            }
        } else {
#pragma unroll
            for (int i = 0; i < NW; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    out[4 * i + j] = minmax_pair_exact((w[i] >> (8 * j + 4)) & 15u, (w[i] >> (8 * j)) & 15u, c);
        }
    } else if (KIND == kInt2) {
        if (c.fast) {
#pragma unroll
            for (int i = 0; i < NW; ++i) {
                uint32_t o[8];
                unpack_int2_word(w[i], o);
#pragma unroll
                for (int j = 0; j < 8; ++j) out[8 * i + j] = hsub_hmul_bf16x2(o[j], c.sub2, c.mul2);
            }
        } else {
#pragma unroll
            for (int i = 0; i < NW; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j)
#pragma unroll
                    for (int h = 0; h < 2; ++h)
                        out[8 * i + 2 * j + h] = minmax_pair_exact((w[i] >> (8 * j + 6 - 4 * h)) & 3u,
                                                                   (w[i] >> (8 * j + 4 - 4 * h)) & 3u, c);
        }
    } else {
        // codebook: W_hat = bf16(fp32(codebook[code] * absmax')), absmax per 64
        const float a = has_dq ? __fadd_rn(__fmul_rn(__fdiv_rn(static_cast<float>(static_cast<int32_t>(pc.a)), 127.0f),
                                                     __uint_as_float(pc.b)),
                                           dq_offset)
                               : __uint_as_float(pc.a);
#pragma unroll
        for (int i = 0; i < NW; ++i)
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
    for (int u0 = 0; u0 < rp; u0 += 16) {
        float b[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) b[u] = (u0 + u < rank) ? bf16_bits_to_f32(__ldg(brow + (u0 + u) * bstride)) : 0.0f;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const float4* t4 = reinterpret_cast<const float4*>(sT + j * rp + u0);
            float d = 0.0f;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const float4 t = t4[v];
                d = fmaf(t.x, b[4 * v], d);
                d = fmaf(t.y, b[4 * v + 1], d);
                d = fmaf(t.z, b[4 * v + 2], d);
                d = fmaf(t.w, b[4 * v + 3], d);
            }
            acc[j] = fmaf(s, d, acc[j]);
        }
    }
}

// Row tt of the adapter operand tile: bf16(s * T[t0 + tt, u]) for u <
// rank_pad in a 128-byte-swizzled K-major tile of 128-byte rows (16-byte
// unit c of row tt at unit c ^ (tt & 7)), zero beyond the rank and beyond the
// mt real tokens.  One token row per thread, its loads all in flight
// together (the tile is staged before the main loop, on its critical path).
__device__ __forceinline__ void stage_scaled_rows(uint8_t* tile, const float* T, int64_t t0, int mt, int nrows,
                                                  int rank, int rank_pad, float s, int tid, int nthreads) {
    for (int tt = tid; tt < nrows; tt += nthreads) {
        const float* row = T + (t0 + tt) * rank;
        const bool tok = tt < mt;
        for (int u0 = 0; u0 < rank_pad; u0 += 16) {
            float v[16];
#pragma unroll
            for (int q = 0; q < 16; ++q) v[q] = (tok && u0 + q < rank) ? __ldg(row + u0 + q) : 0.0f;
            uint32_t w[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) w[q] = pack_bf16x2_rn(__fmul_rn(s, v[2 * q]), __fmul_rn(s, v[2 * q + 1]));
            const int c0 = u0 >> 3;
            *reinterpret_cast<uint4*>(tile + tt * 128 + ((c0 ^ (tt & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
            *reinterpret_cast<uint4*>(tile + tt * 128 + (((c0 + 1) ^ (tt & 7)) << 4)) = make_uint4(w[4], w[5], w[6], w[7]);
        }
    }
}

// Launch shape of the forward kernel: warp 0 = TMA producer, warp 1 = TMEM
// allocator + MMA issuer, then DQW dequantize + epilogue warps.  DQW / 4
// dequant warps share each TMEM lane quarter (warp & 3); part p = (warp-2)/4
// takes part p of every k-block and, in the epilogue, part p of the tokens.
// The 256-token tile (one CTA per SM) runs 16 dequant warps, so that each
// warp's share of a k-block is short and the slowest warp, which gates the
// MMAs, is never far behind; smaller tiles (two CTAs per SM) run 8.
__host__ __device__ constexpr int fwd_threads(int dqw) { return 64 + 32 * dqw; }

__device__ __forceinline__ void tmem_st_32x32b_x8(uint32_t taddr, const uint32_t (&r)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(taddr),
                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
                 : "memory");
}

template <int NT>
struct FwdCfg {
    static constexpr int kXBlocks = NT <= 16 ? 8 : NT <= 32 ? 4 : NT <= 64 ? 2 : 1;   // k-blocks per X box
    static constexpr int kXStages = NT <= 32 ? 2 : NT <= 128 ? 3 : 4;
    static constexpr int kWStages = NT <= 32 ? 4 : NT <= 64 ? 3 : NT <= 128 ? 2 : 4;
    // dequantized A slots in tensor memory: the 256-token tile has room for
    // eight beside its accumulator, so the dequantize warps can run further
    // ahead of the MMAs
    static constexpr int kAStages = NT <= 32 ? 6 : NT >= 256 ? 8 : 4;
    static constexpr int kMinBlocks = NT >= 256 ? 1 : 2;   // CTAs per SM
    static constexpr int kDqWarps = NT >= 256 ? 16 : 8;
};

__device__ __forceinline__ void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

// The output tile a CTA computes: rows n0 .. n0 + 127 of the weight, tokens
// t0 .. t0 + NT - 1, K split `split`; `tile` numbers the tile within its
// GEMM (the split-K counters), `cta` the CTA within the launch (the rotation
// of long k-walks).
struct FwdTile {
    int n0, t0, split;
    uint32_t tile, cta;
};

// One CTA of the forward GEMM (see the top of this file); tmX and tmW are
// the tensor maps of its activations and packed weight.
template <int NT, int KIND, int XS, int XB, int WS, int AS, int DQW>
__device__ __forceinline__ void fwd_tile(const CUtensorMap* tmX, const CUtensorMap* tmW, const FwdParams& p,
                                         const FwdTile tl) {
    constexpr int WB = WeightTile<KIND>::kRowBytes;
    constexpr int PARTS = DQW / 4;                     // dequant warps per TMEM lane quarter
    constexpr int NV = 32 / PARTS;                     // bf16x2 words of a warp's part of a k-block row
    constexpr int SUB = WeightTile<KIND>::kSub;        // k-blocks per weight chunk
    using L = FwdSmem<NT, XS, XB, WS, AS>;
    constexpr int kACols = 32;                         // one k-block of 64 bf16 = 32 columns
    constexpr int kDCol = 0;                           // fp32 accumulator: NT columns
    constexpr int kACol0 = (NT + 31) / 32 * 32;        // A ring after the accumulator
    constexpr uint32_t kTmemCols = tmem_cols_for(kACol0 + kACols * AS);
    static_assert(kACol0 + kACols * AS <= 512, "tensor memory over-subscribed");
    constexpr uint32_t kIdesc = idesc_bf16_f32(128, NT);

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sX = smem + L::kX;
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
    float* s_cb = reinterpret_cast<float*>(smem + L::kMisc + 64);  // 16 floats
    uint8_t* sTop = smem + L::kLoraT;                  // s*T operand tile [NT x 128 B]

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = tl.n0;
    const int t0 = tl.t0;
    const int split = tl.split;
    const int kb_total = p.k / 64;
    const int kb0 = split * p.kb_per_split;            // a multiple of SUB
    const int nkb = min(p.kb_per_split, kb_total - kb0);
    const int nch = (nkb + SUB - 1) / SUB;              // weight chunks of this CTA
    // On long walks (at least 192 k-blocks, K >= 12288) the CTAs of a wave
    // start at different places (a fixed rotation per CTA, in whole weight
    // chunks and activation boxes), so that an activation tile is not first
    // requested by all of them at once; the order of the sum is then fixed
    // per CTA.  (Measured: the 8B down projection at M = 4096 580 -> 545 us;
    // the gate projection, 64 k-blocks, ran slower rotated.)  k-block i of
    // the walk is k-block kbat(i).
    constexpr int RU = SUB > XB ? SUB : XB;
    const int nru = nkb / RU;
    const int rotk = (nkb >= 192 && nkb % RU == 0 && nru > 1)
                         ? static_cast<int>((static_cast<int64_t>(tl.cta) * 37) % nru) * RU
                         : 0;
    auto kbat = [&](int i) { return kb0 + (i + rotk < nkb ? i + rotk : i + rotk - nkb); };
    // the adapter term s * T B^T enters the accumulator through rank/16 MMAs
    // before the main loop, in the first K split only: its A operand (the B
    // rows) takes the first slot of the A ring, as a k-block before the first
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
        tma_prefetch_desc(tmX);
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
    if (threadIdx.x == 0) LBQ_TRACE_EVENT(0, 0);  // kinds: see lbq_trace_read

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        // The weight chunks and the activation tiles are two independent
        // streams: each is issued as soon as its own ring has a free slot
        // (weights: released by the dequantize warps; activations: by the
        // MMAs), so that neither waits behind the other.
        if (lane == 0) {
            const int nxb = (nkb + XB - 1) / XB;           // activation boxes
            int xi = 0, wi = 0;                            // next box / chunk to issue
            ProgressGuard guard;
            bool ok = true;
            while (ok && (wi < nch || xi < nxb)) {
                bool prog = false;
                if (wi < nch && (wi < WS || mbar_try_wait(&emptyW[wi % WS], ((wi / WS) - 1) & 1))) {
                    const int w = wi % WS;
                    mbar_arrive_expect_tx(&fullW[w], L::kWBytes);
                    tma_load_2d(sW + w * L::kWBytes, tmW, &fullW[w], kbat(wi * SUB) * WB, n0);
                    ++wi;
                    prog = true;
                }
                if (xi < nxb && (xi < XS || mbar_try_wait(&emptyX[xi % XS], ((xi / XS) - 1) & 1))) {
                    const int x = xi % XS;
                    LBQ_TRACE_EVENT(6, xi * XB);
                    mbar_arrive_expect_tx(&fullX[x], L::kXBytes);
                    tma_load_3d(sX + x * L::kXBytes, tmX, &fullX[x], 0, t0, kbat(xi * XB));
                    LBQ_TRACE_EVENT(1, xi * XB);
                    ++xi;
                    prog = true;
                }
                ok = guard.step(prog, s_abort);
            }
            // never leave with a copy in flight (matters only after an abort)
            for (int j = max(0, xi - XS); j < xi; ++j) mbar_wait_drain(&fullX[j % XS], (j / XS) & 1);
            for (int c = max(0, wi - WS); c < wi; ++c) mbar_wait_drain(&fullW[c % WS], (c / WS) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            bool ok = true;
            if (lora) {
                // D = (s T) B^T: A = the B rows (A ring slot 0), B operand = s T (shared)
                ok = mbar_wait(&afull[0], 0, s_abort);
                tc_fence_after();
                const uint64_t tdesc = smem_desc_k_sw128(smem_u32(sTop));
                for (int j = 0; ok && j < p.rank_pad / 16; ++j)
                    mma_ts(tmem + kDCol, tmem + kACol0 + 8 * j, tdesc + static_cast<uint64_t>(2 * j), kIdesc,
                           j > 0 ? 1u : 0u);
                if (ok) mma_commit(&aempty[0]);
            }
            for (int i = 0; i < nkb && ok; ++i) {
                const int xj = i / XB, xsub = i - xj * XB, x = xj % XS, ia = i + a_off, a = ia % AS;
                if (xsub == 0) ok = mbar_wait(&fullX[x], (xj / XS) & 1, s_abort);
                LBQ_TRACE_EVENT(4, i);
                ok = ok && mbar_wait(&afull[a], (ia / AS) & 1, s_abort);
                if (!ok) break;
                tc_fence_after();
                LBQ_TRACE_EVENT(5, i);
                const uint64_t bdesc = smem_desc_k_sw128(smem_u32(sX + x * L::kXBytes + xsub * L::kXTile));
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    mma_ts(tmem + kDCol, tmem + kACol0 + a * kACols + 8 * j, bdesc + static_cast<uint64_t>(2 * j), kIdesc,
                           (lora || i > 0 || j > 0) ? 1u : 0u);
                if (xsub == XB - 1 || i == nkb - 1) mma_commit(&emptyX[x]);
                mma_commit(&aempty[a]);
            }
            mma_commit(dfull);  // also completes when nothing was issued
            mbar_wait_drain(dfull, 0);  // MMAs done before tensor memory is freed
        }
    } else {
        // ------------------------------------------------------------ dequantize
        const int q = warp & 3;              // TMEM lane quarter of this warp
        const int part = (warp - 2) >> 2;    // k-block part (and token part in the epilogue)
        const int row = q * 32 + lane;       // output channel within the tile
        const int64_t grow = n0 + row;       // stored weight row
        const bool row_ok = grow < p.n;
        const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
        const bool has_dq = (KIND == kCode4) && (p.q8 != nullptr);
        const float dq_offset = has_dq ? __ldg(p.offset) : 0.0f;
        const int out_col = row_ok ? (p.perm ? p.perm[grow] : static_cast<int>(grow)) : 0;
        const int mt = min(NT, p.m - t0);                  // tokens in this tile
        if (lora) {
            // A operand (ring slot 0): this row's adapter coefficients
            // B[out_col, 2 NV part .. 2 NV part + 2 NV - 1] (bf16, zero beyond the rank)
            uint32_t bv[NV];
#pragma unroll
            for (int i = 0; i < NV; ++i) {
                const int u = 2 * NV * part + 2 * i;
                const uint32_t lo = (row_ok && u < p.rank) ? __ldg(p.B + static_cast<int64_t>(out_col) * p.rank + u) : 0u;
                const uint32_t hi = (row_ok && u + 1 < p.rank) ? __ldg(p.B + static_cast<int64_t>(out_col) * p.rank + u + 1) : 0u;
                bv[i] = lo | (hi << 16);
            }
            if (NV == 16)
                tmem_st_32x32b_x16(tmem + lane_base + kACol0 + NV * part, reinterpret_cast<const uint32_t(&)[16]>(bv));
            else
                tmem_st_32x32b_x8(tmem + lane_base + kACol0 + NV * part, reinterpret_cast<const uint32_t(&)[8]>(bv));
            // B operand: the tile of bf16(s * T) rows
            stage_scaled_rows(sTop, p.T, t0, mt, NT, p.rank, p.rank_pad, p.s, threadIdx.x - 64, 32 * DQW);
            fence_proxy_async_smem();
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&afull[0]);
        }
        // scale and zero (MinMax) change once per group of GB k-blocks, the
        // absmax (codebook) every k-block; loaded one group ahead
        constexpr int GB = (KIND == kInt4) ? 2 : 1;
        PreConst nxt = preload_const<KIND>(p, grow, kbat(0), row_ok && nkb > 0);
        PreConst cur{0u, 0u};
        MinMaxConst mc{};
        // A k-block's tensor-memory store completes while the next k-block is
        // dequantized: its arrival on afull comes one k-block later, off the
        // warp's critical path (the A ring keeps the MMAs fed meanwhile).
        int pend = -1;                                     // A slot whose store is in flight
        auto release_pending = [&]() {
            if (pend < 0) return;
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&afull[pend]);
            pend = -1;
        };
        for (int i = 0; i < nkb; ++i) {
            const int c = i / SUB, sub = i - c * SUB, w = c % WS, ia = i + a_off, a = ia % AS;
            if (i % GB == 0) {
                cur = nxt;
                if (i + GB < nkb) nxt = preload_const<KIND>(p, grow, kbat(i + GB), row_ok);
                if (KIND != kCode4) mc = minmax_const(static_cast<uint16_t>(cur.a), static_cast<uint16_t>(cur.b));
            }
            if (sub == 0 && !mbar_wait(&fullW[w], (c / WS) & 1, s_abort)) break;
            if (ia >= AS && !mbar_wait(&aempty[a], ((ia / AS) - 1) & 1, s_abort)) break;
            tc_fence_after();
            if (lane == 0) LBQ_TRACE_EVENT(2, i * DQW + (warp - 2));
            uint32_t vals[NV];
            if (row_ok) {
                dequant_part_kblock<KIND, NV>(sW + w * L::kWBytes + row * 128, row, sub * WB + part * (WB / PARTS), cur,
                                              mc, dq_offset, has_dq, s_cb, vals);
            } else {
#pragma unroll
                for (int j = 0; j < NV; ++j) vals[j] = 0u;
            }
            // the warp's last read of this weight chunk
            if (sub == SUB - 1 || i == nkb - 1) {
                __syncwarp();
                if (lane == 0) mbar_arrive(&emptyW[w]);
            }
            release_pending();
            if (NV == 16)
                tmem_st_32x32b_x16(tmem + lane_base + kACol0 + a * kACols + NV * part,
                                   reinterpret_cast<const uint32_t(&)[16]>(vals));
            else
                tmem_st_32x32b_x8(tmem + lane_base + kACol0 + a * kACols + NV * part,
                                  reinterpret_cast<const uint32_t(&)[8]>(vals));
            pend = a;
            if (lane == 0) LBQ_TRACE_EVENT(3, i * DQW + (warp - 2));
        }
        release_pending();
        (void)nch;

        // ------------------------------------------------------------ epilogue
        // (the adapter term is already in the accumulator)
        named_barrier_sync(1, 32 * DQW);
        const bool got = mbar_wait(dfull, 0, s_abort);
        tc_fence_after();
        if (threadIdx.x == 64) LBQ_TRACE_EVENT(0, 1);
        const bool splitk = p.nsplit > 1;
        constexpr int kPartCols = NT / PARTS >= 16 ? NT / PARTS : 16;   // token columns per warp part
        const int c_begin = part * kPartCols;
        const int c_end = min(NT, c_begin + kPartCols);
        for (int jj = c_begin; jj < c_end; jj += 16) {
            uint32_t raw[16];
            tmem_ld_32x32b_x16(tmem + lane_base + kDCol + jj, raw);
            tmem_ld_wait();
            if (!row_ok || !got || jj >= mt) continue;
            float acc[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) acc[j] = __uint_as_float(raw[j]);
            if (splitk) {
                float* dst = p.partial + ((static_cast<int64_t>(tl.tile - p.tile0) * p.nsplit + split) * NT + jj) * 128 + row;
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    if (jj + j < mt) dst[j * 128] = acc[j];
                continue;
            }
#pragma unroll
            for (int j = 0; j < 16; ++j)
                if (jj + j < mt) p.Y[static_cast<int64_t>(t0 + jj + j) * p.ldy + out_col] = acc[j];
        }
        if (splitk) {
            // the last CTA of this output tile sums the partials in split order
            __threadfence();
            named_barrier_sync(1, 32 * DQW);
            if (threadIdx.x == 64) {
                const uint32_t tile = tl.tile;
                const uint32_t prev = atomicAdd(p.counters + tile, 1u);
                const int last = (prev == static_cast<uint32_t>(p.nsplit - 1)) ? 1 : 0;
                if (last) p.counters[tile] = 0u;
                *s_last = last;
            }
            named_barrier_sync(1, 32 * DQW);
            if (*s_last && row_ok && got) {
                __threadfence();
                for (int jj = c_begin; jj < min(c_end, mt); jj += 16) {
                    float acc[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) acc[j] = 0.0f;
                    for (int sp = 0; sp < p.nsplit; ++sp) {
                        const float* src =
                            p.partial + ((static_cast<int64_t>(tl.tile - p.tile0) * p.nsplit + sp) * NT + jj) * 128 + row;
                        float part[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) part[j] = (jj + j < mt) ? __ldcg(src + j * 128) : 0.0f;
#pragma unroll
                        for (int j = 0; j < 16; ++j) acc[j] += part[j];
                    }
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        if (jj + j < mt) p.Y[static_cast<int64_t>(t0 + jj + j) * p.ldy + out_col] = acc[j];
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (threadIdx.x == 64) LBQ_TRACE_EVENT(0, 2);
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

template <int NT, int KIND, int XS, int XB, int WS, int AS, int MINB, int DQW>
__global__ void __launch_bounds__(fwd_threads(DQW), MINB)
dqgemm_fwd_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                  const FwdParams p) {
    // a one-dimensional grid: nsplit consecutive CTAs per tile, tiles from
    // tile0 on, row tile fastest
    const int lin = p.tile0 + static_cast<int>(blockIdx.x) / p.nsplit;
    const int split = static_cast<int>(blockIdx.x) % p.nsplit;
    fwd_tile<NT, KIND, XS, XB, WS, AS, DQW>(&tmX, &tmW, p,
                                            FwdTile{(lin % p.rtiles) * 128, (lin / p.rtiles) * NT, split,
                                                    static_cast<uint32_t>(lin), static_cast<uint32_t>(lin)});
}

// A group of forward GEMMs with the same token count in one launch (several
// matrices of a layer, or the two halves of a channel-mix weight): problem i
// owns CTAs cta0[i] .. cta0[i+1]-1, row tiles fastest, then token tiles, and
// no K split.  Every CTA runs the kernel above for its problem's weight kind.
constexpr int kFwdMaxGroup = 8;

struct FwdGroupParams {
    CUtensorMap tmX[kFwdMaxGroup];   // activations of problem i (as for dqgemm_fwd_kernel)
    CUtensorMap tmW[kFwdMaxGroup];   // packed weight of problem i
    FwdParams p[kFwdMaxGroup];
    int kind[kFwdMaxGroup];
    int rtiles[kFwdMaxGroup];        // 128-row tiles of problem i
    int cta0[kFwdMaxGroup + 1];      // first CTA of problem i; cta0[count] = the grid
    int count;
};

template <int NT, int XS, int XB, int WS, int AS, int MINB, int DQW>
__global__ void __launch_bounds__(fwd_threads(DQW), MINB)
dqgemm_fwd_grouped_kernel(const __grid_constant__ FwdGroupParams g) {
    int i = 0;
    for (int j = 1; j < g.count; ++j)
        if (static_cast<int>(blockIdx.x) >= g.cta0[j]) i = j;
    const int local = static_cast<int>(blockIdx.x) - g.cta0[i];
    const FwdTile tl{(local % g.rtiles[i]) * 128, (local / g.rtiles[i]) * NT, 0, static_cast<uint32_t>(local),
                     blockIdx.x};
    if (g.kind[i] == kInt4)
        fwd_tile<NT, kInt4, XS, XB, WS, AS, DQW>(&g.tmX[i], &g.tmW[i], g.p[i], tl);
    else if (g.kind[i] == kInt2)
        fwd_tile<NT, kInt2, XS, XB, WS, AS, DQW>(&g.tmX[i], &g.tmW[i], g.p[i], tl);
    else
        fwd_tile<NT, kCode4, XS, XB, WS, AS, DQW>(&g.tmX[i], &g.tmW[i], g.p[i], tl);
}

}  // namespace lbq
