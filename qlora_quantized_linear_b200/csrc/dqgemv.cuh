// dqgemv.cuh -- bandwidth-bound dequantize-GEMV for decode-sized batches
// (M <= 16 tokens) over a GROUP of weight matrices in one launch.
//
//   Y_i[t, c] = sum_k X_i[t, k] * W_hat_i[c, k]  (+ s_i * sum_u T_i[t, u] B_i[c, u])
//
// At decode sizes the packed weights are the whole cost (0.53 B/param for INT4
// g128), so the kernel is built to stream them once at HBM speed and to pay
// the fixed costs of a launch (start-up, pipeline fill, the tail of split
// tiles) once for a whole layer set instead of once per matrix:
//
//  * persistent, one wave: two CTAs per SM; every CTA gets an equal share
//    (in bytes) of the (128-row tile, 64-wide k-block) work of ONE matrix of
//    the group, contiguous in (tile, k-block) order, so a share may span
//    several tiles;
//  * one producer lane fills a ring of stages.  A stage holds one weight box
//    (128 rows x 128 bytes, 128-byte swizzle, by TMA) and the matching
//    activation slice (a 3-D TMA box of (64 k) x (tokens padded to 8 or 16)
//    x (k-blocks of the weight box), 128-byte swizzle, rows beyond the real
//    tokens read as zeros);
//  * each compute warp copies the per-row constants (scale and zero, or
//    absmax) of its own rows and its part of the box one box ahead with a few
//    cp.async into a double buffer of its own: spread over the eight warps
//    these scattered small reads keep up with the weights, where one producer
//    warp issuing them all for the CTA held the stages back;
//  * eight compute warps.  With up to 8 tokens warp w owns 32 rows (two
//    16-row MMA tiles) and one half of the k-blocks of every box (warps 0-3
//    the first half, 4-7 the second), so a warp's activation fragments and
//    per-token sums serve two row tiles, and at the end of a tile segment the
//    two halves are added in a fixed order through shared memory; with 9..16
//    tokens (twice the accumulators) warp w owns 16 rows and every k-block.
//    Products run on register tensor-core MMAs (mma.sync m16n8k16, bf16 in,
//    fp32 accumulate): rows are the M dimension, tokens (padded to 8 or 16)
//    the N dimension;
//  * codes become bf16 pairs in the cheapest order the packing allows: one
//    logic op turns the two codes that sit two bytes apart in a 32-bit word
//    into a bf16x2 (each half the number 128 + code): 4-bit codes k and k+4,
//    2-bit codes k and k+8.  Each thread puts its activation fragments in
//    the same order with byte permutes (codebook codes pair naturally,
//    through a 256-entry table, and their activations stay as loaded);
//  * dequantization is exact and its scale comes last (GreenBit.AI article,
//    模型量化 (1): one scale and one zero per group): with up to 8 tokens the
//    MMA runs on A = 128 + code (exact in bf16) and, per group, the fold takes
//    (128 + zero) * sum(x) off each token's fp32 partial before multiplying by
//    the scale, the per-token sums coming from MMAs with an all-ones A (the
//    tensor pipe has room for them at this size); with 9..16 tokens A =
//    (128 + code) - (128 + zero) = code - zero in bf16 (exact for |zero| <=
//    128; a group where some row's zero is farther out takes bf16((code -
//    zero) * scale) from fp32 instead).  The codebook format uses
//    bf16(codebook[code]) times the fp32 per-64 absmax (QLoRA explainer,
//    关键技术细节 1);
//  * a tile covered by several CTAs is finished by the one that covers its
//    last k-block (the highest CTA index among them): the others store their
//    fp32 partial sums, count themselves on a per-tile flag and go on; the
//    finishing CTA processes that tile last, waits for the count (CTAs start
//    in index order, so its contributors are running or done, and each of
//    them processes its contributing segment first) and adds the partials in
//    CTA order, so the result does not depend on scheduling.
#pragma once

#include <type_traits>

#include "dqgemm.cuh"

namespace lbq {

constexpr int kGvComputeWarps = 8;                            // 32 rows and half of each box each
constexpr int kGvThreads = 32 * (kGvComputeWarps + 1);        // + one producer warp
constexpr int kGvMaxProblems = 8;                             // matrices per launch
constexpr int kGvMaxStages = 4;
constexpr int kGvWBox = 128 * 128;                            // weight box bytes
constexpr int kGvExtraSmem = 2 * kGvMaxStages * 8 + 16 + 2 * 256 * 4;   // barriers, flags, codebook tables
constexpr int kGvXchgBytes = 4 * 32 * 4 * 4;                  // half the warps' 16x8 fp32 tiles (up to 8 tokens)

// One matrix of a grouped launch (everything but its tensor maps).  Each CTA
// copies its matrix's descriptor into shared memory once, so that the loops
// read it from there.
struct GvProblem {
    const uint16_t* X;                // [m, k] bf16
    float* Y;                         // Y[t * ldy + out_col]
    const int32_t* perm;              // stored row -> output column (NULL = identity)
    const uint16_t* scale;            // [n, ngroups] fp16 (MinMax)
    const uint16_t* zero;             // [n, ngroups] fp16 (MinMax)
    const float* absmax;              // [n * kbt] (codebook, no double quant)
    const int8_t* q8;                 // [n * kbt] (codebook, double quant)
    const float* s2;                  // [ceil(n * kbt / 256)]
    const float* offset;              // [1]
    const float* codebook;            // [16]
    const float* T;                   // [m, rank] fp32
    const uint16_t* B;                // [n_out, rank] bf16, by output column
    float* partial;                   // [ctas + tiles][m][128] fp32 (split tiles)
    uint32_t* counters;               // [tiles] arrival flags, zero at launch and left at zero
    int64_t ldy;
    int64_t total;                    // tiles * kbt  (< 2^31)
    int n, k, kind, ngroups, kbt, tiles, share, cta0, rank;
    int xbytes;                       // bytes of one activation box
    float s;
    int pad_;
};

struct GvParams {
    CUtensorMap tmW[kGvMaxProblems];  // packed weights [n, k*bits/8] u8, box 128 x 128 B, 128-byte swizzle
    CUtensorMap tmX[kGvMaxProblems];  // X as (64, m, k/64) bf16, box (64, 8 or 16, k-blocks per weight box)
    GvProblem prob[kGvMaxProblems];
    int nprob;
    int m;                            // tokens, 1..16
    int ws;                           // ring stages (2..4)
    int stage_bytes;                  // a multiple of 1024: weight box, then the activation box
    int cstride;                      // bytes per row of one constant array in a warp's buffer
    int w_early;                      // weights and constants may be read before the previous kernel ends
};

template <int KIND>
struct GvKind {
    static constexpr int kRowBytes = (KIND == kInt2) ? 16 : 32;   // per row per k-block
    static constexpr int kSub = 128 / kRowBytes;                  // k-blocks per weight box
    static constexpr int kGroupBlocks = (KIND == kInt4) ? 2 : 1;  // k-blocks per scale group (codebook: absmax)
};

// D = A B + C (C = D on entry), one m16n8k16 bf16 MMA with fp32 accumulation.
__device__ __forceinline__ void mma_m16n8k16_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                                  uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D = A B (zero accumulator in).
__device__ __forceinline__ void mma_m16n8k16_bf16_first(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                                        uint32_t a3, uint32_t b0, uint32_t b1) {
    const float z = 0.0f;
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%10, %10, %10, %10};"
        : "=f"(c[0]), "=f"(c[1]), "=f"(c[2]), "=f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(z));
}

// a - b on both bf16 halves (exact here: integers of at most 9 bits).
__device__ __forceinline__ uint32_t sub_bf16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ uint2 gv_lds64(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint4 gv_lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint32_t gv_lds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint16_t gv_lds16(uint32_t addr) {
    uint16_t v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}

// The mbarrier receives one arrival once every cp.async this thread issued so
// far has landed (the arrival is one of the barrier's expected count).
__device__ __forceinline__ void cp_async_mbar_arrive_noinc(uint64_t* bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// One segment of a CTA's share: k-blocks [ka, kb) of row tile `tile`.
struct GvSeg {
    int tile, ka, kb;
};

// A CTA's share: units [u0, u1) of (tile, k-block) in tile-major order, over
// row tiles tA..tB.
struct GvShare {
    int64_t u0, u1;
    int tA, tB, nseg, kbt;
};

// Segment si (0 .. nseg-1) in processing order: the share's last tile first
// (where the CTA contributes to a tile that a later CTA finishes), then the
// whole tiles, then the first tile (which this CTA finishes when it does not
// start it).
__device__ __forceinline__ GvSeg gv_segment(const GvShare& sh, int si) {
    GvSeg s;
    s.tile = sh.nseg == 1 ? sh.tA : (si == 0 ? sh.tB : (si == sh.nseg - 1 ? sh.tA : sh.tA + si));
    s.ka = s.tile == sh.tA ? static_cast<int>(sh.u0 - static_cast<int64_t>(sh.tA) * sh.kbt) : 0;
    s.kb = s.tile == sh.tB ? static_cast<int>(sh.u1 - static_cast<int64_t>(sh.tB) * sh.kbt) : sh.kbt;
    return s;
}

// ----------------------------------------------------------------------------
// producer warp
// ----------------------------------------------------------------------------
// One stage: the weight box and the activation box of k-blocks [kbs, kbs +
// kSub) of row tile `tile`, both arriving on `full` (one expected arrival
// plus their bytes), and the box's constants (one arrival per producer lane).
// The weights and constants may be fetched before the previous kernel on the
// stream has finished; the activations only after.
template <int KIND>
__device__ __forceinline__ void gv_issue_weights(const CUtensorMap* tmW, int xbytes, uint8_t* stage, uint64_t* full,
                                                 int tile, int kbs) {
    mbar_arrive_expect_tx(full, kGvWBox + xbytes);
    tma_load_2d(stage, tmW, full, kbs * GvKind<KIND>::kRowBytes, tile * 128);
}

__device__ __forceinline__ void gv_issue_acts(const CUtensorMap* tmX, uint8_t* stage, uint64_t* full, int kbs) {
    tma_load_3d(stage + kGvWBox, tmX, full, 0, 0, kbs);
}

// A walk over the CTA's weight boxes in processing order.
struct GvBoxCursor {
    const GvShare* sh;
    int sub, si, kbs;
    GvSeg sg;
    bool valid;
    __device__ __forceinline__ void start(const GvShare& s, int sub_) {
        sh = &s;
        sub = sub_;
        si = 0;
        valid = s.nseg > 0;
        if (valid) {
            sg = gv_segment(s, 0);
            kbs = sg.ka;
        }
    }
    __device__ __forceinline__ void next() {
        kbs += sub;
        if (kbs >= sg.kb) {
            if (++si < sh->nseg) {
                sg = gv_segment(*sh, si);
                kbs = sg.ka;
            } else {
                valid = false;
            }
        }
    }
};

__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// The constants of one box (k-blocks [kbs, kbs + nk) of row tile `tile`) for
// rows [row0, row0 + nrows) of the tile into a buffer [2 arrays][nrows]
// [cstride]: lane l copies rows l, l + 32, ..., each as the 4-byte words that
// cover the row's entries (MinMax: scale and zero of the box's groups;
// codebook: the box's absmax values, or its q8 bytes and s2 values).  A row's
// entries may start at an odd 2-byte (or 1-byte) position in its first word;
// the readers account for it.
template <int KIND>
__device__ __forceinline__ void gv_fetch_consts(const GvProblem& P, uint32_t slot, int cstride, int tile, int kbs,
                                                int nk, int row0, int nrows, int lane) {
    constexpr int GB = GvKind<KIND>::kGroupBlocks;
    const uint32_t arr1 = static_cast<uint32_t>(nrows * cstride);   // second array
#pragma unroll 1
    for (int r = lane; r < nrows; r += 32) {
        const int64_t grow = static_cast<int64_t>(tile) * 128 + row0 + r;
        if (grow >= P.n) break;                              // rows ascend with r
        const uint32_t d = slot + r * cstride;
        if (KIND != kCode4) {
            const int64_t e0 = grow * P.ngroups + kbs / GB;
            const int nw = static_cast<int>(((e0 + (nk + GB - 1) / GB - 1) >> 1) - (e0 >> 1)) + 1;
            const uint32_t* sc = reinterpret_cast<const uint32_t*>(P.scale) + (e0 >> 1);
            const uint32_t* ze = reinterpret_cast<const uint32_t*>(P.zero) + (e0 >> 1);
            for (int w = 0; w < nw; ++w) {
                cp_async4(d + 4 * w, sc + w);
                cp_async4(d + arr1 + 4 * w, ze + w);
            }
        } else if (P.q8 == nullptr) {
            const float* src = P.absmax + grow * P.kbt + kbs;
            for (int i = 0; i < nk; ++i) cp_async4(d + 4 * i, src + i);
        } else {
            const int64_t e0 = grow * P.kbt + kbs, e1 = e0 + nk - 1;
            const uint32_t* q32 = reinterpret_cast<const uint32_t*>(P.q8);
            cp_async4(d, q32 + (e0 >> 2));
            if ((e1 >> 2) != (e0 >> 2)) cp_async4(d + 4, q32 + (e1 >> 2));
            cp_async4(d + arr1, P.s2 + (e0 >> 8));
            if ((e1 >> 8) != (e0 >> 8)) cp_async4(d + arr1 + 4, P.s2 + (e1 >> 8));
        }
    }
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

// The producer lane issues the TMA copies; the ring runs ws boxes ahead of
// the compute warps.
template <int KIND>
__device__ __forceinline__ void gv_produce(const GvParams& p, const GvProblem& P, const CUtensorMap* tmW,
                                           const CUtensorMap* tmX, const GvShare& sh, uint8_t* ring, uint64_t* full,
                                           uint64_t* empty, volatile int* s_abort) {
    constexpr int SUB = GvKind<KIND>::kSub;
    const int ws = p.ws;
    GvBoxCursor ic;                                          // next box to issue
    ic.start(sh, SUB);
    int nissued = 0;
    if (p.w_early) {
        // the first boxes' weights before the previous kernel on the stream
        // has finished; the activations only after it has
        GvBoxCursor pre = ic;
        for (int c = 0; pre.valid && c < ws; ++c, pre.next())
            gv_issue_weights<KIND>(tmW, P.xbytes, ring + c * p.stage_bytes, &full[c], pre.sg.tile, pre.kbs);
        griddep_wait();
        for (; ic.valid && nissued < ws; ++nissued, ic.next())
            gv_issue_acts(tmX, ring + nissued * p.stage_bytes, &full[nissued], ic.kbs);
    } else {
        griddep_wait();
        for (; ic.valid && nissued < ws; ++nissued, ic.next()) {
            gv_issue_weights<KIND>(tmW, P.xbytes, ring + nissued * p.stage_bytes, &full[nissued], ic.sg.tile, ic.kbs);
            gv_issue_acts(tmX, ring + nissued * p.stage_bytes, &full[nissued], ic.kbs);
        }
    }
    // box j goes into slot j % ws once the compute warps have released box j - ws
    int slot = 0;
    uint32_t ph = 0;
    for (; ic.valid; ++nissued, ic.next()) {
        if (!mbar_wait(&empty[slot], ph, s_abort)) break;
        uint8_t* stage = ring + slot * p.stage_bytes;
        gv_issue_weights<KIND>(tmW, P.xbytes, stage, &full[slot], ic.sg.tile, ic.kbs);
        gv_issue_acts(tmX, stage, &full[slot], ic.kbs);
        if (++slot == ws) {
            slot = 0;
            ph ^= 1u;
        }
    }
    // never leave with a copy in flight (matters only after an abort)
    for (int i = max(0, nissued - ws); i < nissued; ++i) mbar_wait_drain(&full[i % ws], (i / ws) & 1);
}

// ----------------------------------------------------------------------------
// compute warps
// ----------------------------------------------------------------------------
// bf16 pair of code pair word v (each half 128 + code) with the exact
// fp32 dequantization, rounded once: bf16((code - zero) * scale).
__device__ __forceinline__ uint32_t gv_exact_pair(uint32_t v, float zf, float sf) {
    const float lo = __fmul_rn(__fsub_rn(static_cast<float>(v & 0x7Fu), zf), sf);
    const float hi = __fmul_rn(__fsub_rn(static_cast<float>((v >> 16) & 0x7Fu), zf), sf);
    return pack_bf16x2_rn(lo, hi);
}

template <int KIND, int NT8>
__device__ __forceinline__ void gv_compute(const GvParams& p, const GvProblem& P, const GvShare& sh, int b,
                                           uint8_t* ring, uint8_t* cbuf, uint64_t* full, uint64_t* empty,
                                           volatile int* s_abort, float* xchg, const uint32_t* s_lut,
                                           const float* s_q8lut) {
    using G = GvKind<KIND>;
    constexpr int SUB = G::kSub, RB = G::kRowBytes, GB = G::kGroupBlocks;
    // row tiles per warp and parts of a box's k-blocks: with up to 8 tokens
    // two tiles and two halves, with more one tile and the whole box
    constexpr int TILES = NT8 == 1 ? 2 : 1, KSPLIT = NT8 == 1 ? 2 : 1;
    constexpr int HALF = SUB / KSPLIT;                 // k-blocks of a box per warp
    constexpr int WPK = kGvComputeWarps / KSPLIT;      // warps per k-part
    constexpr int NR = 2 * TILES;                      // rows per thread
    constexpr int TB = RB / 4;                         // code bytes per thread, row and k-block
    constexpr int MPAD = NT8 * 8;                      // token rows of an activation box
    // MinMax with up to 8 tokens: A = 128 + code, the zero folded at the group's end
    constexpr bool kFold = KIND != kCode4 && NT8 == 1;
    // accumulator chains per row tile (two where the fold or the MMA latency wants them)
    constexpr int CH = NT8 == 1 ? 2 : 1;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int j = lane & 3;                            // quarter of the row's bytes
    const int g = lane >> 2;                           // MMA row in the 8-row half, token in the n8 tile
    const int kh = warp / WPK;                         // part of every box's k-blocks
    const int m = p.m;
    // MMA row g is box row pi(g) of the warp's rows (pi interleaves even
    // rows into lanes 0-15 and odd rows into lanes 16-31, so that each half
    // warp's 8-byte reads of the 128-byte-swizzled lines hit 32 distinct
    // banks); the thread's rows are rq, rq + 8 (tile 0) and, with two tiles,
    // rq + 16, rq + 24 (tile 1)
    const int lr0 = (g & 3) * 2 + (g >> 2);
    const int rq = (warp % WPK) * (16 * TILES) + lr0;
    const int sw = rq & 7;                             // swizzle of all four rows' lines
    uint32_t offs[HALF];                               // this thread's bytes of the warp's k-blocks
#pragma unroll
    for (int h = 0; h < HALF; ++h) {
        const int off = (kh * HALF + h) * RB + TB * j;
        offs[h] = static_cast<uint32_t>((((off >> 4) ^ sw) << 4) | (off & 15));
    }
    // B fragments of token nt * 8 + g (a zero row beyond the real tokens):
    // row (s * MPAD + token) of the activation box, 16-byte units 2j and
    // 2j + 1 of its 128-byte line, swizzled with the row (s * MPAD is a
    // multiple of 8, so the swizzle is the token's)
    uint32_t xoff[NT8];
#pragma unroll
    for (int nt = 0; nt < NT8; ++nt) {
        const int tok = nt * 8 + g;
        xoff[nt] = static_cast<uint32_t>(kGvWBox + (kh * HALF * MPAD + tok) * 128 + (((2 * j) ^ (tok & 7)) << 4));
    }
    const float dq_off = (KIND == kCode4 && P.q8 != nullptr) ? __ldg(P.offset) : 0.0f;
    const uint32_t ones = 0x3F803F80u;                       // bf16x2 (1, 1)
    uint32_t mg = 0x43004300u;                               // bf16x2 (128, 128), kept in a register
    asm volatile("" : "+r"(mg));
    const uint32_t cstride = static_cast<uint32_t>(p.cstride);
    // this warp's constant double buffer: [slot][2 arrays][its rows][cstride]
    constexpr int NRW = 16 * TILES;                    // the warp's rows
    const int row0 = (warp % WPK) * NRW;
    const uint32_t arr1 = NRW * cstride;
    const uint32_t cslot_bytes = 2 * NRW * cstride;
    const uint32_t cslot0 = smem_u32(cbuf) + warp * 2 * cslot_bytes;
    // the constants of the warp's part of a box (k-blocks [kbs + kh HALF,
    // kbs + min(nk, (kh + 1) HALF))), for its own rows
    auto fetch_part = [&](uint32_t slot, int tile, int kbs, int nk) {
        const int lo = kh * HALF;
        if (lo < nk) gv_fetch_consts<KIND>(P, slot, p.cstride, tile, kbs + lo, min(nk, lo + HALF) - lo, row0, NRW, lane);
    };
    // the first box's constants; nothing global is written before the
    // previous kernel on the stream has finished
    {
        const GvSeg s0 = gv_segment(sh, 0);
        if (!p.w_early) griddep_wait();
        fetch_part(cslot0, s0.tile, s0.ka, min(SUB, s0.kb - s0.ka));
        cp_async_commit();
        if (p.w_early) griddep_wait();
    }

    bool live = true;                                        // false after a timed-out wait
    int w = 0;                                               // ring slot of the box (matches the producer)
    uint32_t ph = 0;                                         // ... and its phase parity
    uint32_t cbit = 0;                                       // constant slot of the box
    // (after a timed-out wait every warp still runs every segment's barriers)
    for (int si = 0; si < sh.nseg; ++si) {
        const GvSeg sg = gv_segment(sh, si);
        const int tile = sg.tile;
        float acc[TILES][NT8][4];
#pragma unroll
        for (int t2 = 0; t2 < TILES; ++t2)
#pragma unroll
            for (int nt = 0; nt < NT8; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[t2][nt][e] = 0.0f;
        for (int kbs = sg.ka; kbs < sg.kb; kbs += SUB) {
            // the next box's constants into the other slot
            if (kbs + SUB < sg.kb) {
                fetch_part(cslot0 + (cbit ^ 1u) * cslot_bytes, tile, kbs + SUB, min(SUB, sg.kb - kbs - SUB));
            } else if (si + 1 < sh.nseg) {
                const GvSeg sn = gv_segment(sh, si + 1);
                fetch_part(cslot0 + (cbit ^ 1u) * cslot_bytes, sn.tile, sn.ka, min(SUB, sn.kb - sn.ka));
            }
            cp_async_commit();
            cp_async_wait_1();                               // this box's constants (this lane's copies)
            __syncwarp();                                    // ... and the other lanes'
            // warp-uniform: the warp's later shuffles and MMAs need all 32 lanes
            const bool got = live && mbar_wait(&full[w], ph, s_abort);
            live = __all_sync(0xFFFFFFFFu, got);
            const int nk = min(SUB, sg.kb - kbs);
            if (live && kh * HALF < nk) {
                const uint32_t stage = smem_u32(ring + w * p.stage_bytes);
                const uint32_t crow = cslot0 + cbit * cslot_bytes + (rq - row0) * cstride;   // row rq, array 0
                // entry parity of the rows' first constant word (MinMax): the
                // parity of row * groups + first group (the four rows have the
                // parity of rq, as a tile starts on an even row)
                const int s_lo = kh * HALF;                  // the warp's first k-block of the box
                const int par = ((rq & P.ngroups) + (kbs + s_lo) / GB) & 1;
                float sf[NR], zf[NR];
#pragma unroll
                for (int i = 0; i < NR; ++i) {
                    sf[i] = 1.0f;
                    zf[i] = 0.0f;
                }
                bool far = false;
                float cg[TILES][CH][NT8][4], sx[CH][NT8][4];
#pragma unroll
                for (int h = 0; h < HALF; ++h) {
                    const int s = kh * HALF + h;               // k-block of the box
                    if (s < nk) {
                        if (s % GB == 0) {
                            // the group's (or k-block's) constants of the thread's rows
                            if (KIND != kCode4) {
                                const uint32_t ce = crow + 2 * ((s - s_lo) / GB + par);
#pragma unroll
                                for (int i = 0; i < NR; ++i) {
                                    sf[i] = f16_bits_to_f32(gv_lds16(ce + 8 * i * cstride));
                                    zf[i] = f16_bits_to_f32(gv_lds16(ce + 8 * i * cstride + arr1));
                                }
                                if (kFold) {
#pragma unroll
                                    for (int i = 0; i < NR; ++i) zf[i] += 128.0f;   // A = 128 + code
                                } else {
                                    bool f = false;
#pragma unroll
                                    for (int i = 0; i < NR; ++i) f = f || fabsf(zf[i]) > 128.0f;
                                    far = __any_sync(0xFFFFFFFFu, f);
                                }
                            } else if (P.q8 == nullptr) {
#pragma unroll
                                for (int i = 0; i < NR; ++i)
                                    sf[i] = __uint_as_float(gv_lds32(crow + 8 * i * cstride + 4 * (s - s_lo)));
                            } else {
                                // absmax' = fp32(fp32(q8 / 127) * s2) + offset
#pragma unroll
                                for (int i = 0; i < NR; ++i) {
                                    const int64_t e0 = (static_cast<int64_t>(tile) * 128 + rq + 8 * i) * P.kbt + kbs + s_lo;
                                    const int ia = static_cast<int>((e0 & 3) + (s - s_lo));
                                    const uint32_t qa = gv_lds32(crow + 8 * i * cstride + (ia & ~3));
                                    const uint32_t q8 = (qa >> (8 * (ia & 3))) & 0xFFu;
                                    const float s2 = __uint_as_float(
                                        gv_lds32(crow + 8 * i * cstride + arr1 + (((e0 + s - s_lo) >> 8) != (e0 >> 8) ? 4 : 0)));
                                    sf[i] = __fadd_rn(__fmul_rn(s_q8lut[q8], s2), dq_off);
                                }
                            }
                        }
                        // activation fragments of this k-block, in the code pairs' order
                        uint32_t xb[NT8][8];
#pragma unroll
                        for (int nt = 0; nt < NT8; ++nt) {
                            const uint32_t xa = stage + xoff[nt] + h * MPAD * 128;
                            const uint4 lo = gv_lds128(xa);
                            const uint4 hi = gv_lds128(xa ^ 16u);
                            if (KIND == kInt4) {
                                // within each 8 features: (1,5) (0,4) (3,7) (2,6)
                                xb[nt][0] = __byte_perm(lo.x, lo.z, 0x7632);
                                xb[nt][1] = __byte_perm(lo.x, lo.z, 0x5410);
                                xb[nt][2] = __byte_perm(lo.y, lo.w, 0x7632);
                                xb[nt][3] = __byte_perm(lo.y, lo.w, 0x5410);
                                xb[nt][4] = __byte_perm(hi.x, hi.z, 0x7632);
                                xb[nt][5] = __byte_perm(hi.x, hi.z, 0x5410);
                                xb[nt][6] = __byte_perm(hi.y, hi.w, 0x7632);
                                xb[nt][7] = __byte_perm(hi.y, hi.w, 0x5410);
                            } else if (KIND == kInt2) {
                                // within each 16 features: (t, t + 8)
                                xb[nt][0] = __byte_perm(lo.x, hi.x, 0x5410);
                                xb[nt][1] = __byte_perm(lo.x, hi.x, 0x7632);
                                xb[nt][2] = __byte_perm(lo.y, hi.y, 0x5410);
                                xb[nt][3] = __byte_perm(lo.y, hi.y, 0x7632);
                                xb[nt][4] = __byte_perm(lo.z, hi.z, 0x5410);
                                xb[nt][5] = __byte_perm(lo.z, hi.z, 0x7632);
                                xb[nt][6] = __byte_perm(lo.w, hi.w, 0x5410);
                                xb[nt][7] = __byte_perm(lo.w, hi.w, 0x7632);
                            } else {
                                xb[nt][0] = lo.x;
                                xb[nt][1] = lo.y;
                                xb[nt][2] = lo.z;
                                xb[nt][3] = lo.w;
                                xb[nt][4] = hi.x;
                                xb[nt][5] = hi.y;
                                xb[nt][6] = hi.z;
                                xb[nt][7] = hi.w;
                            }
                        }
#pragma unroll
                        for (int t2 = 0; t2 < TILES; ++t2) {
                            // this k-block's codes of the tile's two rows, as bf16x2 pairs
                            const uint32_t wa = stage + (rq + 16 * t2) * 128 + offs[h];
                            uint32_t f0[8], f1[8];
                            if (KIND == kInt4) {
                                const uint2 v0 = gv_lds64(wa);
                                const uint2 v1 = gv_lds64(wa + 1024);
                                int4_pairs(v0.x, mg, f0);
                                int4_pairs(v0.y, mg, f0 + 4);
                                int4_pairs(v1.x, mg, f1);
                                int4_pairs(v1.y, mg, f1 + 4);
                            } else if (KIND == kInt2) {
                                int2_pairs(gv_lds32(wa), mg, f0);
                                int2_pairs(gv_lds32(wa + 1024), mg, f1);
                            } else {
                                const uint2 v0 = gv_lds64(wa);
                                const uint2 v1 = gv_lds64(wa + 1024);
#pragma unroll
                                for (int q = 0; q < 4; ++q) {
                                    f0[q] = s_lut[__byte_perm(v0.x, 0u, 0x4440 + q)];
                                    f0[4 + q] = s_lut[__byte_perm(v0.y, 0u, 0x4440 + q)];
                                    f1[q] = s_lut[__byte_perm(v1.x, 0u, 0x4440 + q)];
                                    f1[4 + q] = s_lut[__byte_perm(v1.y, 0u, 0x4440 + q)];
                                }
                            }
                            if (KIND != kCode4 && !kFold) {
                                if (!far) {
                                    // (128 + code) - (128 + zero) = code - zero exactly
                                    const float z0 = 128.0f + zf[2 * t2], z1 = 128.0f + zf[2 * t2 + 1];
                                    const uint32_t sub0 = pack_bf16x2_rn(z0, z0), sub1 = pack_bf16x2_rn(z1, z1);
#pragma unroll
                                    for (int q = 0; q < 8; ++q) {
                                        f0[q] = sub_bf16x2(f0[q], sub0);
                                        f1[q] = sub_bf16x2(f1[q], sub1);
                                    }
                                } else {
#pragma unroll
                                    for (int q = 0; q < 8; ++q) {
                                        f0[q] = gv_exact_pair(f0[q], zf[2 * t2], sf[2 * t2]);
                                        f1[q] = gv_exact_pair(f1[q], zf[2 * t2 + 1], sf[2 * t2 + 1]);
                                    }
                                }
                            }
#pragma unroll
                            for (int tau = 0; tau < 4; ++tau)
#pragma unroll
                                for (int nt = 0; nt < NT8; ++nt) {
                                    if (s % GB == 0 && tau < CH)
                                        mma_m16n8k16_bf16_first(cg[t2][tau % CH][nt], f0[2 * tau], f1[2 * tau],
                                                                f0[2 * tau + 1], f1[2 * tau + 1], xb[nt][2 * tau],
                                                                xb[nt][2 * tau + 1]);
                                    else
                                        mma_m16n8k16_bf16(cg[t2][tau % CH][nt], f0[2 * tau], f1[2 * tau],
                                                          f0[2 * tau + 1], f1[2 * tau + 1], xb[nt][2 * tau],
                                                          xb[nt][2 * tau + 1]);
                                }
                        }
                        if (kFold) {
                            // per-token sums of the group's activations (every row alike),
                            // in the same chains as the group partials
#pragma unroll
                            for (int tau = 0; tau < 4; ++tau) {
                                if (s % GB == 0 && tau < CH)
                                    mma_m16n8k16_bf16_first(sx[tau % CH][0], ones, ones, ones, ones, xb[0][2 * tau],
                                                            xb[0][2 * tau + 1]);
                                else
                                    mma_m16n8k16_bf16(sx[tau % CH][0], ones, ones, ones, ones, xb[0][2 * tau],
                                                      xb[0][2 * tau + 1]);
                            }
                        }
                        // end of a scale group: fold the group partials
                        if (s % GB == GB - 1 || s == nk - 1) {
#pragma unroll
                            for (int t2 = 0; t2 < TILES; ++t2)
#pragma unroll
                                for (int nt = 0; nt < NT8; ++nt)
#pragma unroll
                                    for (int e = 0; e < 4; ++e) {
                                        const int i = 2 * t2 + (e >> 1);
                                        float cge = cg[t2][0][nt][e];
                                        if (CH == 2) cge += cg[t2][CH - 1][nt][e];
                                        if (kFold) {
                                            const float sxe = sx[0][0][e] + sx[CH - 1][0][e];
                                            acc[t2][nt][e] = fmaf(sf[i], fmaf(-zf[i], sxe, cge), acc[t2][nt][e]);
                                        } else {
                                            acc[t2][nt][e] = fmaf(far ? 1.0f : sf[i], cge, acc[t2][nt][e]);
                                        }
                                    }
                        }
                    }
                }
            }
            // release the slot only after every loaded word has been used
            if (live) {
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[w]);
            }
            if (++w == p.ws) {
                w = 0;
                ph ^= 1u;
            }
            cbit ^= 1u;
        }
        // -------------------------------------------------------------- segment epilogue
        // With two k-parts: warps 0-3 finish tile 0 of their 32 rows, warps
        // 4-7 tile 1, each sum taken as first half + second half.
        float v[NT8][4];
        if (KSPLIT == 1) {
#pragma unroll
            for (int nt = 0; nt < NT8; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) v[nt][e] = acc[0][nt][e];
        } else {
            float* buf = xchg + (warp % WPK) * (32 * 4 * NT8);
            if (kh == 1) {
#pragma unroll
                for (int nt = 0; nt < NT8; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) buf[(nt * 4 + e) * 32 + lane] = acc[0][nt][e];
            }
            asm volatile("bar.sync 1, 256;" ::: "memory");
            if (kh == 0) {
#pragma unroll
                for (int nt = 0; nt < NT8; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) v[nt][e] = acc[0][nt][e] + buf[(nt * 4 + e) * 32 + lane];
            }
            asm volatile("bar.sync 1, 256;" ::: "memory");
            if (kh == 0) {
#pragma unroll
                for (int nt = 0; nt < NT8; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) buf[(nt * 4 + e) * 32 + lane] = acc[TILES - 1][nt][e];
            }
            asm volatile("bar.sync 1, 256;" ::: "memory");
            if (kh == 1) {
#pragma unroll
                for (int nt = 0; nt < NT8; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) v[nt][e] = buf[(nt * 4 + e) * 32 + lane] + acc[TILES - 1][nt][e];
            }
        }
        // this warp's finished rows rl0, rl0 + 8 of the tile
        const int rl0 = rq + 16 * (KSPLIT == 2 ? kh : 0);
        const int64_t gr0 = static_cast<int64_t>(tile) * 128 + rl0, gr1 = gr0 + 8;
        const bool ok0 = gr0 < P.n, ok1 = gr1 < P.n;
        auto lora = [&](int t, int oc) -> float {
            if (P.rank == 0) return 0.0f;
            float d = 0.0f;
            for (int u = 0; u < P.rank; ++u)
                d = fmaf(P.T[static_cast<int64_t>(t) * P.rank + u],
                         bf16_bits_to_f32(__ldg(P.B + static_cast<int64_t>(oc) * P.rank + u)), d);
            return P.s * d;
        };
        if (sg.ka == 0 && sg.kb == P.kbt) {
            // this CTA covered the whole tile
#pragma unroll
            for (int nt = 0; nt < NT8; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int t = nt * 8 + 2 * j + (e & 1);
                    const bool ok = (e < 2) ? ok0 : ok1;
                    const int64_t r = (e < 2) ? gr0 : gr1;
                    if (ok && t < m) {
                        const int oc = P.perm ? P.perm[r] : static_cast<int>(r);
                        P.Y[static_cast<int64_t>(t) * P.ldy + oc] = v[nt][e] + lora(t, oc);
                    }
                }
            continue;
        }
        // split tile.  Partial slot of (CTA b, tile t) is b + t: CTAs cover the
        // work in order, so no two (CTA, tile) pairs share a slot.
        const int cta_lo = static_cast<int>((static_cast<int64_t>(tile) * P.kbt) / P.share);
        const int cta_hi = static_cast<int>((static_cast<int64_t>(tile + 1) * P.kbt - 1) / P.share);
        if (sg.kb < P.kbt) {
            // contributor (the tile's last k-block belongs to a later CTA)
            float* slot = P.partial + (static_cast<int64_t>(b) + tile) * m * 128;
#pragma unroll
            for (int nt = 0; nt < NT8; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int t = nt * 8 + 2 * j + (e & 1);
                    if (t < m) slot[t * 128 + rl0 + ((e < 2) ? 0 : 8)] = v[nt][e];
                }
            asm volatile("bar.sync 1, 256;" ::: "memory");
            if (tid == 0) flag_publish(P.counters + tile);
            continue;
        }
        // this CTA finishes the tile: wait for the cta_hi - cta_lo contributors
        if (tid == 0) {
            if (!flag_wait_geq(P.counters + tile, static_cast<uint32_t>(cta_hi - cta_lo))) *s_abort = 1;
            P.counters[tile] = 0u;                          // left at zero for the next call
        }
        asm volatile("bar.sync 1, 256;" ::: "memory");
        // the contributors' partials in CTA order (QB CTAs' loads in flight
        // together), then this CTA's own sums
        constexpr int QB = NT8 == 1 ? 8 : 4;
        float u[NT8][4];
#pragma unroll
        for (int nt = 0; nt < NT8; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) u[nt][e] = 0.0f;
        for (int b0 = cta_lo; b0 < cta_hi; b0 += QB) {
            float part[QB][NT8][4];
#pragma unroll
            for (int q = 0; q < QB; ++q)
#pragma unroll
                for (int nt = 0; nt < NT8; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int t = nt * 8 + 2 * j + (e & 1);
                        part[q][nt][e] = (b0 + q < cta_hi && t < m)
                                             ? __ldcg(P.partial + ((static_cast<int64_t>(b0 + q) + tile) * m + t) * 128 +
                                                      rl0 + ((e < 2) ? 0 : 8))
                                             : 0.0f;
                    }
#pragma unroll
            for (int q = 0; q < QB; ++q)
#pragma unroll
                for (int nt = 0; nt < NT8; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) u[nt][e] += part[q][nt][e];
        }
#pragma unroll
        for (int nt = 0; nt < NT8; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int t = nt * 8 + 2 * j + (e & 1);
                const bool ok = (e < 2) ? ok0 : ok1;
                const int64_t r = (e < 2) ? gr0 : gr1;
                if (ok && t < m) {
                    const int oc = P.perm ? P.perm[r] : static_cast<int>(r);
                    P.Y[static_cast<int64_t>(t) * P.ldy + oc] = (u[nt][e] + v[nt][e]) + lora(t, oc);
                }
            }
    }
    cp_async_wait_all();                                     // no copy into the buffer outlives the CTA
}

template <int NT8>
__global__ void __launch_bounds__(kGvThreads, 2) dqgemv_grouped_kernel(const __grid_constant__ GvParams p) {
    // let the next kernel on the stream be scheduled as soon as our CTAs leave
    griddep_launch_dependents();
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    // this CTA's matrix and its index among that matrix's CTAs; its
    // descriptor goes to shared memory once
    int pi = 0;
    for (int i = 1; i < p.nprob; ++i)
        if (static_cast<int>(blockIdx.x) >= p.prob[i].cta0) pi = i;
    __shared__ GvProblem s_prob;
    {
        static_assert(sizeof(GvProblem) % 4 == 0, "descriptor copied in words");
        const uint32_t* src = reinterpret_cast<const uint32_t*>(&p.prob[pi]);
        uint32_t* dst = reinterpret_cast<uint32_t*>(&s_prob);
        for (int i = tid; i < static_cast<int>(sizeof(GvProblem) / 4); i += kGvThreads) dst[i] = src[i];
    }
    __syncthreads();
    const GvProblem& P = s_prob;
    const int b = static_cast<int>(blockIdx.x) - P.cta0;

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte alignment for the swizzled boxes, by pointer arithmetic on the
    // shared array so that every access below stays a shared-memory access
    uint8_t* ring = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* cbuf = ring + p.ws * p.stage_bytes;                               // [warp][2][2][rows][cstride]
    float* xchg = reinterpret_cast<float*>(cbuf + kGvComputeWarps * 2 * 2 * (16 * (3 - NT8)) * p.cstride);   // [4][4][32]
    uint64_t* full = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(xchg) + (NT8 == 1 ? kGvXchgBytes : 0));
    uint64_t* empty = full + kGvMaxStages;
    volatile int* s_abort = reinterpret_cast<volatile int*>(empty + kGvMaxStages);
    uint32_t* s_lut = reinterpret_cast<uint32_t*>(empty + kGvMaxStages) + 4;   // codebook pairs [256]
    float* s_q8lut = reinterpret_cast<float*>(s_lut + 256);                  // q8 / 127 [256]

    // the share: units [u0, u1) of (tile, k-block), in tile-major order
    GvShare sh;
    sh.kbt = P.kbt;
    sh.u0 = static_cast<int64_t>(b) * P.share;
    sh.u1 = min(sh.u0 + P.share, P.total);
    sh.tA = static_cast<int>(sh.u0 / P.kbt);
    sh.tB = sh.u0 < sh.u1 ? static_cast<int>((sh.u1 - 1) / P.kbt) : sh.tA - 1;
    sh.nseg = sh.tB - sh.tA + 1;

    if (tid == kGvComputeWarps * 32) {
        tma_prefetch_desc(&p.tmW[pi]);
        tma_prefetch_desc(&p.tmX[pi]);
        for (int i = 0; i < p.ws; ++i) {
            mbar_init(&full[i], 1);                      // the producer's TMA arrival + the boxes' bytes
            mbar_init(&empty[i], kGvComputeWarps);
        }
        *s_abort = 0;
        fence_mbar_init();
    }
    if (P.kind == kCode4) {
        for (int e = tid; e < 256; e += kGvThreads) {
            // byte e = (first code << 4) | second code -> (codebook[first], codebook[second])
            s_lut[e] = pack_bf16x2_rn(__ldg(P.codebook + (e >> 4)), __ldg(P.codebook + (e & 15)));
            s_q8lut[e] = __fdiv_rn(static_cast<float>(static_cast<int8_t>(static_cast<uint8_t>(e))), 127.0f);
        }
    }
    __syncthreads();
    if (sh.nseg <= 0) return;

    auto run = [&](auto kind_tag) {
        constexpr int KIND = decltype(kind_tag)::value;
        if (warp == kGvComputeWarps) {
            if (lane == 0) gv_produce<KIND>(p, P, &p.tmW[pi], &p.tmX[pi], sh, ring, full, empty, s_abort);
        } else {
            gv_compute<KIND, NT8>(p, P, sh, b, ring, cbuf, full, empty, s_abort, xchg, s_lut, s_q8lut);
        }
    };
    if (P.kind == kInt4)
        run(std::integral_constant<int, kInt4>{});
    else if (P.kind == kInt2)
        run(std::integral_constant<int, kInt2>{});
    else
        run(std::integral_constant<int, kCode4>{});
}

}  // namespace lbq
