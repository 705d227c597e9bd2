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
//  * one producer lane fills a ring of stages, each with two TMA copies: one
//    weight box (128 rows x 128 bytes, 128-byte swizzle) and the matching
//    activation slice, a 3-D box of (64 k) x (tokens padded to 8 or 16) x
//    (k-blocks of the weight box), 128-byte swizzle (rows beyond the real
//    tokens read as zeros).  No prologue stages a CTA's whole slice first;
//  * each compute warp fetches the per-row constants (scale and zero, or
//    absmax) of its own 16 rows one weight box ahead, with a few cp.async
//    into a small buffer of its own, so the constants never wait on memory
//    and the producer stays a single lane;
//  * eight compute warps own 16 rows each; a thread owns two rows (r, r+8)
//    and, per k-block, 16 consecutive codes of each.  Products run on
//    register tensor-core MMAs (mma.sync m16n8k16, bf16 in, fp32 accumulate):
//    rows are the M dimension, tokens (padded to 8 or 16) the N dimension;
//  * codes become bf16 pairs in the cheapest order the packing allows: one
//    logic op turns the two codes that sit two bytes apart in a 32-bit word
//    into a bf16x2 (each half the number 128 + code): 4-bit codes k and k+4,
//    2-bit codes k and k+8.  The producer warp's lanes permute each landed
//    activation box in place to the same order (codebook codes pair
//    naturally, through a 256-entry table, and their activations stay as
//    loaded), then release the stage to the compute warps on a second barrier;
//  * dequantization is exact and its scale comes last (GreenBit.AI article,
//    模型量化 (1): one scale and one zero per group): with up to 8 tokens the
//    MMA runs on A = 128 + code (exact in bf16) and, per group, the fold takes
//    (128 + zero) * sum(x) off each token's fp32 partial before multiplying by
//    the scale, the per-token sums coming from MMAs with an all-ones A (the
//    tensor pipe has room for them at this size); with 9..16 tokens A =
//    (128 + code) - (128 + zero) = code - zero in bf16 (exact for |zero| <=
//    128; a group where some row's zero is farther out falls back to the
//    folded form).  The codebook format uses bf16(codebook[code]) times the
//    fp32 per-64 absmax (QLoRA explainer, 关键技术细节 1);
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

constexpr int kGvComputeWarps = 8;                            // 16 rows each: 128 rows per tile
constexpr int kGvThreads = 32 * (kGvComputeWarps + 1);        // + one producer warp
constexpr int kGvMaxProblems = 8;                             // matrices per launch
constexpr int kGvMaxStages = 4;
constexpr int kGvWBox = 128 * 128;                            // weight box bytes
constexpr int kGvExtraSmem = 3 * kGvMaxStages * 8 + 16 + 2 * 256 * 4;   // barriers, flags, codebook tables
constexpr int kGvConstWords = 5;                              // 4-byte words per row and array a box needs (max)

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

// Calls fn(box index, tile, first k-block, k-blocks) for the CTA's weight
// boxes in processing order until fn returns false.  The producer and the
// compute warps walk the same sequence.
template <int SUB, typename F>
__device__ __forceinline__ void gv_for_each_box(const GvShare& sh, F&& fn) {
    int c = 0;
    for (int si = 0; si < sh.nseg; ++si) {
        const GvSeg sg = gv_segment(sh, si);
        for (int kbs = sg.ka; kbs < sg.kb; kbs += SUB, ++c)
            if (!fn(c, sg.tile, kbs, min(SUB, sg.kb - kbs))) return;
    }
}

// ----------------------------------------------------------------------------
// producer lane
// ----------------------------------------------------------------------------
// One stage: the weight box and the activation box of k-blocks [kbs, kbs +
// kSub) of row tile `tile`, both arriving on `full` (one expected arrival
// plus their bytes).  The weights (and the arrival) may be issued before the
// previous kernel on the stream has finished; the activations only after.
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

// Puts the activations of a landed box (the m real token rows of its kSub
// k-blocks) in the order of the weight-code pairs: within 8 consecutive k
// (4-bit) the pairs (1,5) (0,4) (3,7) (2,6); within 16 (2-bit) the pairs
// (t, t+8).  Rows are 128-byte lines swizzled with the token (kSub * 8 or
// 16 rows per k-block, so the row's swizzle is the token's).
template <int KIND>
__device__ __forceinline__ void gv_permute_acts(uint8_t* xbox, int m, int mpad, int lane) {
    constexpr int SUB = GvKind<KIND>::kSub;
    const uint32_t base = smem_u32(xbox);
    for (int s = 0; s < SUB; ++s) {
        if (KIND == kInt4) {
            for (int e = lane; e < m * 8; e += 32) {
                const int t = e >> 3, u = e & 7;
                const uint32_t a = base + (s * mpad + t) * 128 + ((u ^ (t & 7)) << 4);
                const uint4 v = gv_lds128(a);
                const uint4 o = make_uint4(__byte_perm(v.x, v.z, 0x7632), __byte_perm(v.x, v.z, 0x5410),
                                           __byte_perm(v.y, v.w, 0x7632), __byte_perm(v.y, v.w, 0x5410));
                asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(o.x), "r"(o.y), "r"(o.z),
                             "r"(o.w)
                             : "memory");
            }
        } else {
            for (int e = lane; e < m * 4; e += 32) {
                const int t = e >> 2, up = e & 3;
                const uint32_t row = base + (s * mpad + t) * 128;
                const uint32_t a0 = row + (((2 * up) ^ (t & 7)) << 4), a1 = row + (((2 * up + 1) ^ (t & 7)) << 4);
                const uint4 v = gv_lds128(a0), w = gv_lds128(a1);
                const uint4 o0 = make_uint4(__byte_perm(v.x, w.x, 0x5410), __byte_perm(v.x, w.x, 0x7632),
                                            __byte_perm(v.y, w.y, 0x5410), __byte_perm(v.y, w.y, 0x7632));
                const uint4 o1 = make_uint4(__byte_perm(v.z, w.z, 0x5410), __byte_perm(v.z, w.z, 0x7632),
                                            __byte_perm(v.w, w.w, 0x5410), __byte_perm(v.w, w.w, 0x7632));
                asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a0), "r"(o0.x), "r"(o0.y), "r"(o0.z),
                             "r"(o0.w)
                             : "memory");
                asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a1), "r"(o1.x), "r"(o1.y), "r"(o1.z),
                             "r"(o1.w)
                             : "memory");
            }
        }
    }
}

// The producer warp: lane 0 issues the TMA copies, kept ws boxes ahead; the
// warp permutes each box's activations once it has landed and releases the
// stage on xready.  Box c's slot is refilled (with box c + ws) once the
// compute warps have released it, after box c + 1 has been released to them.
template <int KIND>
__device__ __forceinline__ void gv_produce(const GvParams& p, const CUtensorMap* tmW, const CUtensorMap* tmX,
                                           int xbytes, const GvShare& sh, uint8_t* ring, uint64_t* full,
                                           uint64_t* xready, uint64_t* empty, volatile int* s_abort, int lane) {
    constexpr int SUB = GvKind<KIND>::kSub;
    const int ws = p.ws, mpad = p.m <= 8 ? 8 : 16;
    GvBoxCursor ic;                                          // next box to issue
    ic.start(sh, SUB);
    int nissued = 0;
    if (p.w_early) {
        // the ring's weights before the previous kernel on the stream has
        // finished; the activations only after it has
        GvBoxCursor pre = ic;
        for (int c = 0; pre.valid && c < ws; ++c, pre.next())
            if (lane == 0) gv_issue_weights<KIND>(tmW, xbytes, ring + c * p.stage_bytes, &full[c], pre.sg.tile, pre.kbs);
        griddep_wait();
        for (; ic.valid && nissued < ws; ++nissued, ic.next())
            if (lane == 0) gv_issue_acts(tmX, ring + nissued * p.stage_bytes, &full[nissued], ic.kbs);
    } else {
        griddep_wait();
        for (; ic.valid && nissued < ws; ++nissued, ic.next()) {
            if (lane == 0) {
                gv_issue_weights<KIND>(tmW, xbytes, ring + nissued * p.stage_bytes, &full[nissued], ic.sg.tile, ic.kbs);
                gv_issue_acts(tmX, ring + nissued * p.stage_bytes, &full[nissued], ic.kbs);
            }
        }
    }
    GvBoxCursor pc;                                          // next box to release
    pc.start(sh, SUB);
    for (int c = 0; pc.valid; ++c, pc.next()) {
        const int w = c % ws;
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&full[w], (c / ws) & 1, s_abort))) break;
        uint8_t* stage = ring + w * p.stage_bytes;
        if (KIND != kCode4) {
            gv_permute_acts<KIND>(stage + kGvWBox, p.m, mpad, lane);
            fence_proxy_async_smem();                        // before the next TMA write to this stage
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&xready[w]);
        if (c >= 1 && ic.valid) {
            const int wp = (c - 1) % ws;
            if (!__all_sync(0xFFFFFFFFu, mbar_wait(&empty[wp], ((c - 1) / ws) & 1, s_abort))) break;
            if (lane == 0) {
                gv_issue_weights<KIND>(tmW, xbytes, ring + wp * p.stage_bytes, &full[wp], ic.sg.tile, ic.kbs);
                gv_issue_acts(tmX, ring + wp * p.stage_bytes, &full[wp], ic.kbs);
            }
            ic.next();
            ++nissued;
        }
    }
    // never leave with a copy in flight (matters only after an abort)
    if (lane == 0)
        for (int i = max(0, nissued - ws); i < nissued; ++i) mbar_wait_drain(&full[i % ws], (i / ws) & 1);
    __syncwarp();
}

// ----------------------------------------------------------------------------
// per-warp constants
// ----------------------------------------------------------------------------
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// The raw constants of one box for the warp's 16 rows into one of its two
// buffer slots: lane (row lr = lane % 16, array lane / 16) copies the 4-byte
// words that cover the row's entries (MinMax: scale, zero; codebook: absmax,
// or q8 and s2).  A row's entries may start at an odd 2-byte (or 1-byte)
// position in its first word; the readers account for it.
template <int KIND>
__device__ __forceinline__ void gv_fetch_consts(const GvProblem& P, uint32_t slot, int cstride, int tile, int kbs,
                                                int nk, int warp, int lane) {
    constexpr int GB = GvKind<KIND>::kGroupBlocks;
    const int lr = lane & 15, arr = lane >> 4;
    const int64_t grow = static_cast<int64_t>(tile) * 128 + warp * 16 + lr;
    if (grow >= P.n) return;
    const uint32_t d = slot + (arr * 16 + lr) * cstride;
    if (KIND != kCode4) {
        const int g0 = kbs / GB, ng = (nk + GB - 1) / GB;
        const int64_t e0 = grow * P.ngroups + g0;
        const uint32_t* src = reinterpret_cast<const uint32_t*>(arr ? P.zero : P.scale);
        const int64_t w0 = e0 >> 1, w1 = (e0 + ng - 1) >> 1;
        for (int64_t w = w0; w <= w1; ++w) cp_async4(d + static_cast<uint32_t>(w - w0) * 4, src + w);
    } else if (P.q8 == nullptr) {
        if (arr == 0) {
            const int64_t e0 = grow * P.kbt + kbs;
            for (int i = 0; i < nk; ++i) cp_async4(d + 4 * i, P.absmax + e0 + i);
        }
    } else {
        const int64_t e0 = grow * P.kbt + kbs, e1 = e0 + nk - 1;
        if (arr == 0) {
            const uint32_t* q32 = reinterpret_cast<const uint32_t*>(P.q8);
            cp_async4(d, q32 + (e0 >> 2));
            if ((e1 >> 2) != (e0 >> 2)) cp_async4(d + 4, q32 + (e1 >> 2));
        } else {
            cp_async4(d, P.s2 + (e0 >> 8));
            if ((e1 >> 8) != (e0 >> 8)) cp_async4(d + 4, P.s2 + (e1 >> 8));
        }
    }
}

// ----------------------------------------------------------------------------
// compute warps
// ----------------------------------------------------------------------------
template <int KIND, int NT8>
__device__ __forceinline__ void gv_compute(const GvParams& p, const GvProblem& P, const GvShare& sh, int b,
                                           uint8_t* ring, uint64_t* xready, uint64_t* empty, volatile int* s_abort,
                                           uint8_t* cbuf, const uint32_t* s_lut, const float* s_q8lut) {
    using G = GvKind<KIND>;
    constexpr int SUB = G::kSub, RB = G::kRowBytes, GB = G::kGroupBlocks;
    constexpr int TB = RB / 4;                         // code bytes per thread, row and k-block
    constexpr int MPAD = NT8 * 8;                      // token rows of an activation box
    // MinMax with up to 8 tokens: A = 128 + code, the zero folded at the group's end
    constexpr bool kFold = KIND != kCode4 && NT8 == 1;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int j = lane & 3;                            // quarter of the row's bytes
    const int g = lane >> 2;                           // MMA row in the 8-row half, token in the n8 tile
    const int m = p.m;
    // MMA row g is weight row pi(g) of the warp's first 8 (pi interleaves even
    // rows into lanes 0-15 and odd rows into lanes 16-31, so that each half
    // warp's 8-byte reads of the 128-byte-swizzled lines hit 32 distinct banks)
    const int lr0 = (g & 3) * 2 + (g >> 2);                 // warp-local rows lr0, lr0 + 8
    const int rl0 = warp * 16 + lr0;                        // tile rows rl0, rl0 + 8
    const int sw = rl0 & 7;                                 // swizzle of both rows' lines
    uint32_t offs[SUB];                                     // this thread's bytes of k-block s in the line
#pragma unroll
    for (int s = 0; s < SUB; ++s) {
        const int off = s * RB + TB * j;
        offs[s] = static_cast<uint32_t>((((off >> 4) ^ sw) << 4) | (off & 15));
    }
    // B fragments of token nt * 8 + g (a zero row beyond the real tokens):
    // row (s * MPAD + token) of the activation box, 16-byte units 2j and
    // 2j + 1 of its 128-byte line, swizzled with the row (s * MPAD is a
    // multiple of 8, so the swizzle is the token's)
    uint32_t xoff[NT8];
#pragma unroll
    for (int nt = 0; nt < NT8; ++nt) {
        const int tok = nt * 8 + g;
        xoff[nt] = static_cast<uint32_t>(kGvWBox + tok * 128 + (((2 * j) ^ (tok & 7)) << 4));
    }
    const float dq_off = (KIND == kCode4 && P.q8 != nullptr) ? __ldg(P.offset) : 0.0f;
    const uint32_t ones = 0x3F803F80u;                       // bf16x2 (1, 1)
    uint32_t mg = 0x43004300u;                               // bf16x2 (128, 128), kept in a register
    asm volatile("" : "+r"(mg));
    // this warp's two constant slots; rows lr0 and lr0 + 8 of array 0 / 1
    const uint32_t cslot0 = smem_u32(cbuf) + warp * (2 * 32 * p.cstride);
    const uint32_t cslot_bytes = 32 * p.cstride;
    const uint32_t zoff = 16 * p.cstride;

    // the first box's constants; nothing global is written before the
    // previous kernel on the stream has finished
    {
        const GvSeg s0 = gv_segment(sh, 0);
        if (!p.w_early) griddep_wait();
        gv_fetch_consts<KIND>(P, cslot0, p.cstride, s0.tile, s0.ka, min(SUB, s0.kb - s0.ka), warp, lane);
        cp_async_commit();
        if (p.w_early) griddep_wait();
    }

    bool live = true;                                        // false after a timed-out wait
    int c = 0;                                               // boxes consumed (matches the producer)
    // (after a timed-out wait every warp still runs every segment's barriers)
    for (int si = 0; si < sh.nseg; ++si) {
        const GvSeg sg = gv_segment(sh, si);
        const int tile = sg.tile;
        const int64_t gr0 = static_cast<int64_t>(tile) * 128 + rl0, gr1 = gr0 + 8;
        const bool ok0 = gr0 < P.n, ok1 = gr1 < P.n;
        // per-token activation sums sx; with the folded zero they are kept in
        // the same two chains as the group partials cg, so that (128 + zero)
        // * sum(x) cancels the code-independent part of cg exactly when 128 +
        // zero is a power of two (an all-zero row gives exactly 0)
        constexpr int SXC = kFold ? 2 : 1;
        float acc[NT8][4], cg[2][NT8][4], sx[SXC][NT8][4];
#pragma unroll
        for (int nt = 0; nt < NT8; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                acc[nt][e] = cg[0][nt][e] = cg[1][nt][e] = 0.0f;
#pragma unroll
                for (int ch = 0; ch < SXC; ++ch) sx[ch][nt][e] = 0.0f;
            }
        for (int kbs = sg.ka; kbs < sg.kb; kbs += SUB, ++c) {
            // the next box's constants into the other slot
            if (kbs + SUB < sg.kb) {
                gv_fetch_consts<KIND>(P, cslot0 + ((c + 1) & 1) * cslot_bytes, p.cstride, tile, kbs + SUB,
                                      min(SUB, sg.kb - kbs - SUB), warp, lane);
            } else if (si + 1 < sh.nseg) {
                const GvSeg sn = gv_segment(sh, si + 1);
                gv_fetch_consts<KIND>(P, cslot0 + ((c + 1) & 1) * cslot_bytes, p.cstride, sn.tile, sn.ka,
                                      min(SUB, sn.kb - sn.ka), warp, lane);
            }
            cp_async_commit();
            cp_async_wait_1();                               // this box's constants (this lane's copies)
            __syncwarp();                                    // ... and the other lanes'
            const int w = c % p.ws;
            // warp-uniform: the warp's later shuffles and MMAs need all 32 lanes
            const bool got = live && mbar_wait(&xready[w], (c / p.ws) & 1, s_abort);
            live = __all_sync(0xFFFFFFFFu, got);
            if (!live) continue;
            const int nk = min(SUB, sg.kb - kbs);
            const uint32_t stage = smem_u32(ring + w * p.stage_bytes);
            const uint32_t wrow = stage + rl0 * 128;
            const uint32_t cs = cslot0 + (c & 1) * cslot_bytes;
            const uint32_t ca0 = cs + lr0 * p.cstride, ca1 = cs + (lr0 + 8) * p.cstride;
            // entry parity of the rows' first constant word (MinMax)
            int par0 = 0, par1 = 0;
            if (KIND != kCode4) {
                const int g0 = kbs / GB;
                par0 = static_cast<int>((gr0 * P.ngroups + g0) & 1);
                par1 = static_cast<int>((gr1 * P.ngroups + g0) & 1);
            }
            uint32_t sub0 = 0x43004300u, sub1 = 0x43004300u;
            float sf0 = 1.0f, sf1 = 1.0f, zf0 = 0.0f, zf1 = 0.0f;
            bool far = false;
#pragma unroll
            for (int s = 0; s < SUB; ++s) {
                if (s < nk) {
                    if (s % GB == 0) {
                        if (KIND != kCode4) {
                            const int gi = s / GB;
                            sf0 = f16_bits_to_f32(gv_lds16(ca0 + 2 * (gi + par0)));
                            sf1 = f16_bits_to_f32(gv_lds16(ca1 + 2 * (gi + par1)));
                            zf0 = f16_bits_to_f32(gv_lds16(ca0 + zoff + 2 * (gi + par0)));
                            zf1 = f16_bits_to_f32(gv_lds16(ca1 + zoff + 2 * (gi + par1)));
                            if (kFold) {
                                // A = 128 + code: the fold takes (128 + zero) * sum(x) off
                                zf0 += 128.0f;
                                zf1 += 128.0f;
                                far = true;
                            } else {
                                far = __any_sync(0xFFFFFFFFu, (fabsf(zf0) > 128.0f) || (fabsf(zf1) > 128.0f));
                            }
                            if (kFold) {
                            } else if (far) {
                                // A = code (exact); zero * sum(x) is taken off at the fold
                                sub0 = sub1 = 0x43004300u;
                            } else {
                                // (128 + code) - (128 + zero) = code - zero exactly
                                sub0 = pack_bf16x2_rn(128.0f + zf0, 128.0f + zf0);
                                sub1 = pack_bf16x2_rn(128.0f + zf1, 128.0f + zf1);
                            }
                        } else if (P.q8 == nullptr) {
                            sf0 = __uint_as_float(gv_lds32(ca0 + 4 * s));
                            sf1 = __uint_as_float(gv_lds32(ca1 + 4 * s));
                        } else {
                            // absmax' = fp32(fp32(q8 / 127) * s2) + offset
                            const int64_t e0a = gr0 * P.kbt + kbs, e0b = gr1 * P.kbt + kbs;
                            const int ia = static_cast<int>((e0a & 3) + s), ib = static_cast<int>((e0b & 3) + s);
                            const uint32_t qa = gv_lds32(ca0 + (ia & ~3)), qb = gv_lds32(ca1 + (ib & ~3));
                            const uint32_t q8a = (qa >> (8 * (ia & 3))) & 0xFFu, q8b = (qb >> (8 * (ib & 3))) & 0xFFu;
                            const float s2a = __uint_as_float(gv_lds32(ca0 + zoff + (((e0a + s) >> 8) != (e0a >> 8) ? 4 : 0)));
                            const float s2b = __uint_as_float(gv_lds32(ca1 + zoff + (((e0b + s) >> 8) != (e0b >> 8) ? 4 : 0)));
                            sf0 = __fadd_rn(__fmul_rn(s_q8lut[q8a], s2a), dq_off);
                            sf1 = __fadd_rn(__fmul_rn(s_q8lut[q8b], s2b), dq_off);
                        }
                    }
                    // this k-block's codes of the thread's two rows, as bf16x2 pairs
                    uint32_t f0[8], f1[8];
                    if (KIND == kInt4) {
                        const uint2 v0 = gv_lds64(wrow + offs[s]);
                        const uint2 v1 = gv_lds64(wrow + 1024 + offs[s]);
                        int4_pairs(v0.x, mg, f0);
                        int4_pairs(v0.y, mg, f0 + 4);
                        int4_pairs(v1.x, mg, f1);
                        int4_pairs(v1.y, mg, f1 + 4);
                    } else if (KIND == kInt2) {
                        int2_pairs(gv_lds32(wrow + offs[s]), mg, f0);
                        int2_pairs(gv_lds32(wrow + 1024 + offs[s]), mg, f1);
                    } else {
                        const uint2 v0 = gv_lds64(wrow + offs[s]);
                        const uint2 v1 = gv_lds64(wrow + 1024 + offs[s]);
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            f0[q] = s_lut[__byte_perm(v0.x, 0u, 0x4440 + q)];
                            f0[4 + q] = s_lut[__byte_perm(v0.y, 0u, 0x4440 + q)];
                            f1[q] = s_lut[__byte_perm(v1.x, 0u, 0x4440 + q)];
                            f1[4 + q] = s_lut[__byte_perm(v1.y, 0u, 0x4440 + q)];
                        }
                    }
                    if (KIND != kCode4 && !kFold) {
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            f0[q] = sub_bf16x2(f0[q], sub0);
                            f1[q] = sub_bf16x2(f1[q], sub1);
                        }
                    }
                    // B fragments: the 16 activations of the thread's quarter
                    // (steps 0, 1 from the first 16 bytes, 2, 3 from the next)
                    uint32_t xb[NT8][8];
#pragma unroll
                    for (int nt = 0; nt < NT8; ++nt) {
                        const uint32_t xa = stage + xoff[nt] + s * MPAD * 128;
                        const uint4 lo = gv_lds128(xa);
                        const uint4 hi = gv_lds128(xa ^ 16u);
                        xb[nt][0] = lo.x;
                        xb[nt][1] = lo.y;
                        xb[nt][2] = lo.z;
                        xb[nt][3] = lo.w;
                        xb[nt][4] = hi.x;
                        xb[nt][5] = hi.y;
                        xb[nt][6] = hi.z;
                        xb[nt][7] = hi.w;
                    }
#pragma unroll
                    for (int tau = 0; tau < 4; ++tau)
#pragma unroll
                        for (int nt = 0; nt < NT8; ++nt) {
                            if (s % GB == 0 && tau < 2)
                                mma_m16n8k16_bf16_first(cg[tau & 1][nt], f0[2 * tau], f1[2 * tau], f0[2 * tau + 1],
                                                        f1[2 * tau + 1], xb[nt][2 * tau], xb[nt][2 * tau + 1]);
                            else
                                mma_m16n8k16_bf16(cg[tau & 1][nt], f0[2 * tau], f1[2 * tau], f0[2 * tau + 1],
                                                  f1[2 * tau + 1], xb[nt][2 * tau], xb[nt][2 * tau + 1]);
                        }
                    if (KIND != kCode4 && far) {
                        // per-token sums of the group's activations (every row alike)
#pragma unroll
                        for (int tau = 0; tau < 4; ++tau)
#pragma unroll
                            for (int nt = 0; nt < NT8; ++nt) {
                                if (s % GB == 0 && tau < SXC)
                                    mma_m16n8k16_bf16_first(sx[tau % SXC][nt], ones, ones, ones, ones, xb[nt][2 * tau],
                                                            xb[nt][2 * tau + 1]);
                                else
                                    mma_m16n8k16_bf16(sx[tau % SXC][nt], ones, ones, ones, ones, xb[nt][2 * tau],
                                                      xb[nt][2 * tau + 1]);
                            }
                    }
                    // end of a scale group: fold the group partial
                    if (s % GB == GB - 1 || s == nk - 1) {
                        if (KIND != kCode4 && far) {
#pragma unroll
                            for (int nt = 0; nt < NT8; ++nt) {
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const float sxe = SXC == 2 ? sx[0][nt][e] + sx[SXC - 1][nt][e] : sx[0][nt][e];
                                    const float cge = cg[0][nt][e] + cg[1][nt][e];
                                    acc[nt][e] = fmaf(e < 2 ? sf0 : sf1, fmaf(e < 2 ? -zf0 : -zf1, sxe, cge), acc[nt][e]);
                                }
                            }
                        } else {
#pragma unroll
                            for (int nt = 0; nt < NT8; ++nt) {
                                acc[nt][0] = fmaf(sf0, cg[0][nt][0] + cg[1][nt][0], acc[nt][0]);
                                acc[nt][1] = fmaf(sf0, cg[0][nt][1] + cg[1][nt][1], acc[nt][1]);
                                acc[nt][2] = fmaf(sf1, cg[0][nt][2] + cg[1][nt][2], acc[nt][2]);
                                acc[nt][3] = fmaf(sf1, cg[0][nt][3] + cg[1][nt][3], acc[nt][3]);
                            }
                        }
                    }
                }
            }
            // release the slot only after every loaded word has been used
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[w]);
        }
        // -------------------------------------------------------------- segment epilogue
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
                        P.Y[static_cast<int64_t>(t) * P.ldy + oc] = acc[nt][e] + lora(t, oc);
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
                    if (t < m) slot[t * 128 + rl0 + ((e < 2) ? 0 : 8)] = acc[nt][e];
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
        float v[NT8][4];
#pragma unroll
        for (int nt = 0; nt < NT8; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) v[nt][e] = 0.0f;
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
                    for (int e = 0; e < 4; ++e) v[nt][e] += part[q][nt][e];
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
                    P.Y[static_cast<int64_t>(t) * P.ldy + oc] = (v[nt][e] + acc[nt][e]) + lora(t, oc);
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
    uint8_t* cbuf = ring + p.ws * p.stage_bytes;                              // [warp][slot][array][16 rows]
    uint64_t* full = reinterpret_cast<uint64_t*>(cbuf + kGvComputeWarps * 2 * 32 * p.cstride);
    uint64_t* xready = full + kGvMaxStages;
    uint64_t* empty = xready + kGvMaxStages;
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
            mbar_init(&full[i], 1);                      // the producer's arrival + the boxes' bytes
            mbar_init(&xready[i], 1);                    // activations in the pairs' order
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
        if (warp == kGvComputeWarps)
            gv_produce<KIND>(p, &p.tmW[pi], &p.tmX[pi], P.xbytes, sh, ring, full, xready, empty, s_abort, lane);
        else
            gv_compute<KIND, NT8>(p, P, sh, b, ring, xready, empty, s_abort, cbuf, s_lut, s_q8lut);
    };
    if (P.kind == kInt4)
        run(std::integral_constant<int, kInt4>{});
    else if (P.kind == kInt2)
        run(std::integral_constant<int, kInt2>{});
    else
        run(std::integral_constant<int, kCode4>{});
}

}  // namespace lbq
