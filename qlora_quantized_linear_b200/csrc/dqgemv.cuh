// dqgemv.cuh -- bandwidth-bound dequantize-GEMV for decode-sized batches
// (M <= 16 tokens), stream-K over (row tile, k-block) work.
//
//   Y[t, c] = sum_k X[t, k] * W_hat[c, k]  (+ s * sum_u T[t, u] B[c, u])
//
// At decode sizes the packed weight is the whole cost (0.53 B/param for INT4
// g128), so the kernel is built to stream it once at HBM speed:
//
//  * one producer lane streams the CTA's weight rows through a ring of
//    128-row x 128-byte TMA boxes (128-byte swizzle); large boxes keep the TMA
//    engine efficient and the ring keeps ~64 KB per CTA in flight without any
//    load instruction in the compute warps;
//  * eight compute warps own 16 rows each; a thread owns two rows (r, r+8)
//    and, per 64-wide k-block, a quarter of each row's bytes.  Products run on
//    register-resident tensor-core MMAs (mma.sync m16n8k16, bf16 in, fp32
//    accumulate): rows are the M dimension, tokens (padded to 8 or 16) the N
//    dimension;
//  * codes become bf16 with one mask-and-or per two codes (the bf16 number
//    128 + code), pairing codes that sit 2 bytes apart; the k order inside an
//    MMA step is whatever pairing the codes have, and the activations staged in
//    shared memory are permuted the same way, so each activation fragment is
//    one 8-byte load;
//  * dequantization is exact: A = bf16(code - zero) (exact for |zero| <= 128;
//    otherwise bf16(code) with -zero * sum(x) added per group) and the
//    per-group scale multiplies the fp32 group partial after the group's MMAs
//    (GreenBit.AI article, 模型量化 (1): a scale and a zero per group).  The
//    codebook format uses bf16(codebook[code]) times the fp32 per-64 absmax
//    (QLoRA explainer, 关键技术细节 1).  Each (row, group) constant is
//    converted once per CTA into a shared-memory table at the start, not by
//    every lane that uses it;
//  * stream-K: the grid is a whole number of waves and every CTA gets an equal
//    contiguous share of the (row tile, k-block) work, spanning at most two
//    row tiles.  A tile covered by several CTAs is finished by the one that
//    covers its last k-block (the highest CTA index among them): the others
//    store their partial sums, count themselves on a per-tile flag and leave
//    without waiting; the finishing CTA waits for the count (CTAs start in
//    index order, so its contributors are running or done) and adds the
//    partials in CTA order, so the result does not depend on scheduling.
#pragma once

#include <type_traits>

#include "dqgemm.cuh"

namespace lbq {

constexpr int kGemvComputeWarps = 8;                            // 16 rows each: 128 rows per tile
constexpr int kGemvThreads = 32 * (kGemvComputeWarps + 1);      // + one producer warp
constexpr int kGemvMaxWStages = 4;                              // 16 KB weight boxes in flight (3 or 4)
constexpr int kGemvTabPerThread = 16;                           // constant-table entries per thread
constexpr int kGemvMaxTabGroups = 2 * kGemvTabPerThread;        // groups (codebook: k-blocks) per CTA

struct GemvParams {
    int m, n, k;                      // tokens, stored rows, input features
    int ngroups;                      // k / group (MinMax)
    const uint16_t* scale;            // [n, ngroups] fp16 (MinMax)
    const uint16_t* zero;             // [n, ngroups] fp16 (MinMax)
    const float* absmax;              // codebook, no double quant
    const int8_t* q8;                 // codebook, double quant
    const float* s2;
    const float* offset;
    const float* codebook;
    const uint16_t* X;                // [m, k] bf16
    int rank;
    float s;
    const float* T;                   // [m, rank]
    const uint16_t* B;                // [n_out, rank]
    float* Y;
    int64_t ldy;
    const int32_t* perm;
    int kbt;                          // k-blocks per row (k / 64)
    int tiles;                        // row tiles of 128
    int share;                        // k-blocks per CTA (<= kbt; a multiple of the scale group)
    int64_t total;                    // tiles * kbt
    float* partial;                   // [grid + tiles][m][128]
    uint32_t* counters;               // [tiles] arrival flags, zero at launch and left at zero
    int w_early;                      // the packed weight and its constants may be read before the
                                      // previous kernel on the stream has finished
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

template <int KIND>
struct GemvTile {
    static constexpr int kRowBytes = (KIND == kInt2) ? 16 : 32;        // per row per k-block
    static constexpr int kThreadBytes = kRowBytes / 4;                 // a quarter row
    static constexpr int kSub = 128 / kRowBytes;                       // k-blocks per weight box
    static constexpr int kGroupBlocks = (KIND == kInt4) ? 2 : 1;       // k-blocks per scale group
    // shared table of per-(group, row) constants, 4 bytes each: MinMax the
    // bf16 subtrahend 128 + zero (low half) and the fp16 scale (high half);
    // codebook the fp32 absmax of each (k-block, row)
    static constexpr int kTabEntry = 4;
};

// Order of the 16 activations of a 16-wide k group as the MMA steps consume
// them: step tau reads four consecutive entries (two code pairs).  4-bit
// MinMax codes pair nibbles two bytes apart (k and k+4 in the group); 2-bit
// codes pair crumbs two bytes apart (k and k+8); codebook codes pair the two
// nibbles of one byte (k and k+1, the natural order).
__device__ __forceinline__ int gemv_xperm(int kind, int p) {
    constexpr int kPerm4[16] = {1, 5, 0, 4, 3, 7, 2, 6, 9, 13, 8, 12, 11, 15, 10, 14};
    constexpr int kPerm2[16] = {0, 8, 1, 9, 2, 10, 3, 11, 4, 12, 5, 13, 6, 14, 7, 15};
    return kind == kInt2 ? kPerm2[p] : kind == kInt4 ? kPerm4[p] : p;
}

// (a & MASK) | c in one logic op.
template <uint32_t MASK>
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t c) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "n"(MASK), "r"(c));
    return d;
}

// Code pairs of one 32-bit word of 4-bit codes (bytes b0..b3 = codes 0..7):
// P0 = (1, 5), P1 = (0, 4), P2 = (3, 7), P3 = (2, 6), each half the bf16
// number 128 + code (mg = 0x43004300 is passed in a register).
__device__ __forceinline__ void int4_pairs(uint32_t w, uint32_t mg, uint32_t* o) {
    o[0] = and_or<0x000F000Fu>(w, mg);
    o[1] = and_or<0x000F000Fu>(w >> 4, mg);
    o[2] = and_or<0x000F000Fu>(w >> 8, mg);
    o[3] = and_or<0x000F000Fu>(w >> 12, mg);
}

// Code pairs of one 32-bit word of 2-bit codes (bytes b0..b3 = codes 0..15,
// first code in the top bits): pair t = (t, t + 8), t = 0..7.
__device__ __forceinline__ void int2_pairs(uint32_t w, uint32_t mg, uint32_t* o) {
    o[0] = and_or<0x00030003u>(w >> 6, mg);
    o[1] = and_or<0x00030003u>(w >> 4, mg);
    o[2] = and_or<0x00030003u>(w >> 2, mg);
    o[3] = and_or<0x00030003u>(w, mg);
    o[4] = and_or<0x00030003u>(w >> 14, mg);
    o[5] = and_or<0x00030003u>(w >> 12, mg);
    o[6] = and_or<0x00030003u>(w >> 10, mg);
    o[7] = and_or<0x00030003u>(w >> 8, mg);
}

// a - b on both bf16 halves (exact here: integers of at most 9 bits).
__device__ __forceinline__ uint32_t sub_bf16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ uint2 gemv_lds64(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint32_t gemv_lds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

// Split-tile flags: a contributor publishes its partial sums (stored by all
// threads of the CTA before the barrier that precedes this call) and counts
// itself; the finishing CTA waits for the count with acquire semantics.
__device__ __forceinline__ void flag_publish(uint32_t* f) {
    asm volatile("fence.acq_rel.gpu;\n\tred.relaxed.gpu.global.add.u32 [%0], 1;" ::"l"(f) : "memory");
}

__device__ __forceinline__ uint32_t flag_load_acquire(const uint32_t* f) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(f) : "memory");
    return v;
}

// Bounded wait for *f >= want; records kStatusTimeout and returns false when
// it gives up.
__device__ __forceinline__ bool flag_wait_geq(const uint32_t* f, uint32_t want) {
    if (flag_load_acquire(f) >= want) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 0; it < kWaitLimitIters; ++it) {
        __nanosleep(64);
        if (flag_load_acquire(f) >= want) return true;
        if ((it & 63u) == 63u && globaltimer_ns() - t0 > kWaitLimitNs) break;
    }
    record_status(kStatusTimeout);
    return false;
}

template <int KIND, int NTOK, int WS>
__global__ void __launch_bounds__(kGemvThreads, 2)
dqgemv_kernel(const __grid_constant__ CUtensorMap tmW, const GemvParams p) {
    constexpr int NT8 = NTOK / 8;
    constexpr int GB = GemvTile<KIND>::kGroupBlocks;
    constexpr int SUB = GemvTile<KIND>::kSub;
    constexpr int RB = GemvTile<KIND>::kRowBytes;
    constexpr int TB = GemvTile<KIND>::kThreadBytes;
    constexpr int TE = GemvTile<KIND>::kTabEntry;
    constexpr int TW = TB / 4;                                    // code words per row, k-block and thread
    static_assert(WS >= 2 && WS <= kGemvMaxWStages, "weight ring depth");
    constexpr int kWBox = 128 * 128;
    constexpr int kCompute = 32 * kGemvComputeWarps;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // let the next kernel on the stream be scheduled as soon as our CTAs leave
    griddep_launch_dependents();
    if (tid == kCompute) tma_prefetch_desc(&tmW);

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // 1024-byte alignment for the swizzled boxes, by pointer arithmetic on the
    // shared array so that every access below stays a shared-memory access
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t* sW = smem;                                           // WS x 16 KB
    const int xstride = p.share * 64 + 4;                         // bf16 per token row (+8 bytes)
    // token rows, plus a zero row m when the token tile has padding lanes
    const int xrows = p.m < NTOK ? p.m + 1 : p.m;
    uint16_t* sX = reinterpret_cast<uint16_t*>(smem + WS * kWBox);          // [xrows][xstride]
    // constant table [128 rows][tstride]: an odd row stride keeps the eight
    // rows that a warp reads at once in distinct banks
    const int tstride = (p.share / GB) | 1;
    uint8_t* sTab = reinterpret_cast<uint8_t*>(sX + xrows * xstride);
    uint32_t* s_lut = reinterpret_cast<uint32_t*>(sTab + 128 * tstride * TE);     // codebook pairs [256]
    uint64_t* full = reinterpret_cast<uint64_t*>(s_lut + (KIND == kCode4 ? 256 : 0));
    uint64_t* empty = full + WS;
    int* s_misc = reinterpret_cast<int*>(empty + WS);
    volatile int* s_abort = s_misc;
    int* s_far = s_misc + 1;

    // this CTA's work: up to two (tile, first k-block, k-blocks) segments
    // (tiles * kbt < 2^31, checked by the host)
    int t0 = 0, a0 = 0, n0 = 0, n1 = 0;
    {
        const uint32_t u0 = blockIdx.x * static_cast<uint32_t>(p.share);
        const uint32_t tot = static_cast<uint32_t>(p.total);
        const uint32_t u1 = u0 + p.share < tot ? u0 + p.share : tot;
        if (u0 < u1) {
            t0 = static_cast<int>(u0 / static_cast<uint32_t>(p.kbt));
            a0 = static_cast<int>(u0 - static_cast<uint32_t>(t0) * p.kbt);
            n0 = min(static_cast<int>(u1 - u0), p.kbt - a0);
            n1 = static_cast<int>(u1 - u0) - n0;
        }
    }
    const int nseg = n0 == 0 ? 0 : (n1 == 0 ? 1 : 2);
    const int nk = n0 + n1;
    // the second segment (the start of tile t0 + 1) is processed first: its
    // partial sums are published before this CTA waits on anything, so the
    // CTAs that finish tiles never wait on each other in a chain
    const int nbox1 = (n1 + SUB - 1) / SUB;
    const int nbox = nbox1 + (n0 + SUB - 1) / SUB;

    // the producer lane issues the first weight box at once; the rest of the
    // ring fills only after the compute threads have issued their loads
    // (small scattered loads queued behind megabytes of weight boxes come
    // back microseconds late)
    auto issue_box = [&](int c) {
        const int w = c % WS;
        mbar_arrive_expect_tx(&full[w], kWBox);
        const int x = c < nbox1 ? c * SUB * RB : (a0 + (c - nbox1) * SUB) * RB;
        const int y = (c < nbox1 ? t0 + 1 : t0) * 128;
        tma_load_2d(sW + w * kWBox, &tmW, &full[w], x, y);
    };
    if (tid == kCompute) {
        for (int i = 0; i < WS; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], kGemvComputeWarps);
        }
        *s_abort = 0;
        *s_far = 0;
        fence_mbar_init();
        if (!p.w_early) griddep_wait();
        if (nbox > 0) issue_box(0);
    }
    // prologue, first half (compute threads): issue the global loads of this
    // CTA's constants and of its first activation round, so that they reach
    // memory ahead of all but the first weight box
    const int ngr16 = nk * 4;                                      // 16-wide k groups of the slice
    const int xtotal = p.m * ngr16;
    constexpr int XU = (KIND == kCode4) ? 2 : 4;                  // activation loads in flight per round
    const int G = nk / GB, G0 = n0 / GB;                           // table groups (codebook: k-blocks)
    // table entry (row rl, group lg) of thread (warp w, lane) and slot u = 2 it + ch:
    // rl = 16 w + 2 it + lane / 16, lg = lane % 16 + 16 ch (coalesced along the row)
    uint32_t raw[kGemvTabPerThread], raw2[kGemvTabPerThread];
    uint4 v[XU][2];
    if (tid < kCompute) {
        // the weight's constants may be read early; the activations (and the
        // workspace, Y, T) only after the previous kernel has finished
        if (!p.w_early) griddep_wait();
#pragma unroll
        for (int u = 0; u < kGemvTabPerThread; ++u) {
            const int rl = 16 * warp + 2 * (u >> 1) + (lane >> 4), lg = (lane & 15) + 16 * (u & 1);
            raw[u] = 0u;
            raw2[u] = 0u;
            if (lg < G) {
                const bool sb = lg >= G0;
                const int64_t r = static_cast<int64_t>(sb ? t0 + 1 : t0) * 128 + rl;
                const int gl = sb ? lg - G0 : a0 / GB + lg;            // group (codebook: k-block) in the row
                // plain loads only: no arithmetic on a loaded value before the
                // barrier below, or the thread would wait for the data there
                if (r < p.n) {
                    if (KIND != kCode4) {
                        raw[u] = __ldg(p.scale + r * p.ngroups + gl);
                        raw2[u] = __ldg(p.zero + r * p.ngroups + gl);
                    } else if (p.q8 != nullptr) {
                        const int64_t bi = r * p.kbt + gl;
                        raw[u] = __ldg(reinterpret_cast<const uint8_t*>(p.q8) + bi);
                        raw2[u] = __float_as_uint(__ldg(p.s2 + (bi >> 8)));
                    } else {
                        raw[u] = __float_as_uint(__ldg(p.absmax + r * p.kbt + gl));
                    }
                }
            }
        }
        if (p.w_early) griddep_wait();
#pragma unroll
        for (int u = 0; u < XU; ++u) {
            const int e = tid + u * kCompute;
            if (e < xtotal) {
                const int t = e / ngr16, g16 = e - t * ngr16;
                const int lk = g16 >> 2;
                const int kb = lk < n0 ? a0 + lk : lk - n0;
                const uint4* src = reinterpret_cast<const uint4*>(p.X + static_cast<int64_t>(t) * p.k + kb * 64 +
                                                                  (g16 & 3) * 16);
                v[u][0] = __ldg(src);
                v[u][1] = __ldg(src + 1);
            }
        }
    }

    __syncthreads();

    if (warp == kGemvComputeWarps) {
        // ------------------------------------------------------------ producer
        if (lane == 0 && nbox > 0) {
            int issued = 1;
            for (int c = 1; c < nbox; ++c) {
                if (c >= WS && !mbar_wait(&empty[c % WS], ((c / WS) - 1) & 1, s_abort)) break;
                issue_box(c);
                issued = c + 1;
            }
            for (int c = max(0, issued - WS); c < issued; ++c) mbar_wait_drain(&full[c % WS], (c / WS) & 1);
        }
        return;
    }

    // ---------------------------------------------------------------- compute warps
    // prologue, second half: store the activations, convert the constants
    // (the empty asm keeps every use of the loaded values after the barrier)
#pragma unroll
    for (int u = 0; u < kGemvTabPerThread; ++u) asm volatile("" : "+r"(raw[u]), "+r"(raw2[u]));
#pragma unroll
    for (int u = 0; u < XU; ++u)
        asm volatile("" : "+r"(v[u][0].x), "+r"(v[u][0].y), "+r"(v[u][0].z), "+r"(v[u][0].w), "+r"(v[u][1].x),
                     "+r"(v[u][1].y), "+r"(v[u][1].z), "+r"(v[u][1].w));
    {
        // activations of the m real tokens, permuted to the MMA step order
        for (int e0 = tid; e0 < xtotal; e0 += XU * kCompute) {
            if (e0 != tid) {
#pragma unroll
                for (int u = 0; u < XU; ++u) {
                    const int e = e0 + u * kCompute;
                    if (e < xtotal) {
                        const int t = e / ngr16, g16 = e - t * ngr16;
                        const int lk = g16 >> 2;
                        const int kb = lk < n0 ? a0 + lk : lk - n0;
                        const uint4* src = reinterpret_cast<const uint4*>(p.X + static_cast<int64_t>(t) * p.k +
                                                                          kb * 64 + (g16 & 3) * 16);
                        v[u][0] = __ldg(src);
                        v[u][1] = __ldg(src + 1);
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < XU; ++u) {
                const int e = e0 + u * kCompute;
                if (e < xtotal) {
                    const int t = e / ngr16, g16 = e - t * ngr16;
                    const uint32_t w8[8] = {v[u][0].x, v[u][0].y, v[u][0].z, v[u][0].w,
                                            v[u][1].x, v[u][1].y, v[u][1].z, v[u][1].w};
                    uint16_t in[16];
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        in[2 * q] = static_cast<uint16_t>(w8[q] & 0xFFFFu);
                        in[2 * q + 1] = static_cast<uint16_t>(w8[q] >> 16);
                    }
                    // rows are 8-byte aligned (stride 128 * share + 8 bytes)
                    uint2* d2 = reinterpret_cast<uint2*>(sX + t * xstride + g16 * 16);
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        d2[q] = make_uint2(static_cast<uint32_t>(in[gemv_xperm(KIND, 4 * q)]) |
                                               (static_cast<uint32_t>(in[gemv_xperm(KIND, 4 * q + 1)]) << 16),
                                           static_cast<uint32_t>(in[gemv_xperm(KIND, 4 * q + 2)]) |
                                               (static_cast<uint32_t>(in[gemv_xperm(KIND, 4 * q + 3)]) << 16));
                }
            }
        }
        // convert the constants into the table
        const float dq_off = (KIND == kCode4 && p.q8 != nullptr) ? __ldg(p.offset) : 0.0f;
#pragma unroll
        for (int u = 0; u < kGemvTabPerThread; ++u) {
            const int rl = 16 * warp + 2 * (u >> 1) + (lane >> 4), lg = (lane & 15) + 16 * (u & 1);
            if (lg < G) {
                if (KIND != kCode4) {
                    const uint16_t s16 = static_cast<uint16_t>(raw[u]), z16 = static_cast<uint16_t>(raw2[u]);
                    const float zf = f16_bits_to_f32(z16);
                    uint32_t word;
                    if (fabsf(zf) <= 128.0f) {
                        // (128 + q) - (128 + z) = q - z exactly
                        word = pack_bf16x2_rn(128.0f + zf, 0.0f) & 0xFFFFu;
                    } else {
                        // (128 + q) - 128 = q; the zero is added after the loop
                        word = 0x4300u;
                        *s_far = 1;
                    }
                    *reinterpret_cast<uint32_t*>(sTab + (rl * tstride + lg) * 4) =
                        word | (static_cast<uint32_t>(s16) << 16);
                } else {
                    float am = __uint_as_float(raw[u]);
                    if (p.q8 != nullptr)
                        am = __fadd_rn(__fmul_rn(__fdiv_rn(static_cast<float>(static_cast<int8_t>(static_cast<uint8_t>(raw[u]))), 127.0f),
                                                 __uint_as_float(raw2[u])),
                                       dq_off);
                    *reinterpret_cast<float*>(sTab + (rl * tstride + lg) * 4) = am;
                }
            }
        }
        // row m: zeros, read by the lanes of tokens >= m
        if (p.m < NTOK)
            for (int e = tid; e < xstride / 2; e += kCompute)
                reinterpret_cast<uint32_t*>(sX + p.m * xstride)[e] = 0u;
        if (KIND == kCode4) {
            for (int e = tid; e < 256; e += kCompute) {
                // byte e = (first code << 4) | second code -> (codebook[first], codebook[second])
                s_lut[e] = pack_bf16x2_rn(p.codebook[e >> 4], p.codebook[e & 15]);
            }
        }
    }
    asm volatile("bar.sync 1, 256;" ::: "memory");

    const int j = lane & 3;                            // quarter of the row's bytes
    const int g = lane >> 2;                           // MMA row in the 8-row half, token in the n8 tile
    // MMA row g is weight row pi(g) of the warp's first 8 (pi interleaves even
    // rows into lanes 0-15 and odd rows into lanes 16-31, so that each half
    // warp's 8-byte reads of the 128-byte-swizzled lines hit 32 distinct banks)
    const int rl0 = warp * 16 + (g & 3) * 2 + (g >> 2); // local rows rl0, rl0 + 8
    const int sw = rl0 & 7;                            // swizzle of both rows' lines
    uint32_t offs[SUB];                                // this thread's bytes of sub-block s in the line
#pragma unroll
    for (int s = 0; s < SUB; ++s) {
        const int off = s * RB + TB * j;
        offs[s] = static_cast<uint32_t>((((off >> 4) ^ sw) << 4) | (off & 15));
    }
    const uint32_t wrow = smem_u32(sW) + rl0 * 128;
    const uint32_t trow = smem_u32(sTab) + rl0 * tstride * TE;   // table row rl0 (row rl0 + 8: + 8 tstride TE)
    // B fragments: token nt * 8 + g; lanes of tokens >= m read the zero row
    // (a select per load would cost more than the loads themselves)
    uint32_t xthr[NT8];
#pragma unroll
    for (int nt = 0; nt < NT8; ++nt) {
        const int tok = nt * 8 + g < p.m ? nt * 8 + g : p.m;
        xthr[nt] = smem_u32(sX) + static_cast<uint32_t>(tok * xstride + 16 * j) * 2;
    }
    const bool far = *s_far != 0;                      // some group of this CTA has |zero| > 128
    uint32_t mg = 0x43004300u;
    asm volatile("" : "+r"(mg));                       // keep the magic in a register

    uint32_t c = 0;                                    // weight boxes consumed (matches the producer)
    // (after a timed-out wait every warp still runs both segments' barriers)
    for (int si = 0; si < nseg; ++si) {
        const int sgi = nseg - 1 - si;                 // segment 1 (if any) first, then segment 0
        const int tile = sgi == 0 ? t0 : t0 + 1;
        const int kb0 = sgi == 0 ? a0 : 0;
        const int nkb = sgi == 0 ? n0 : n1;
        const int lk0 = sgi == 0 ? 0 : n0;             // first local k-block of the segment
        const int64_t gr0 = static_cast<int64_t>(tile) * 128 + rl0, gr1 = gr0 + 8;
        const bool ok0 = gr0 < p.n, ok1 = gr1 < p.n;
        // group partials in two chains (even and odd MMA steps), folded per group
        float acc[NT8][4], cg[2][NT8][4];
#pragma unroll
        for (int nt = 0; nt < NT8; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[nt][e] = cg[0][nt][e] = cg[1][nt][e] = 0.0f;
        uint32_t sub0 = 0x43004300u, sub1 = 0x43004300u;
        float sf0 = 1.0f, sf1 = 1.0f;

        const int nbx = (nkb + SUB - 1) / SUB;
        const int nfull = nkb / SUB;                      // boxes whose SUB k-blocks all belong to the segment
        // one box of k-blocks; the per-k-block bounds test is compiled only
        // into the copy used for a partial last box (it costs ~15% of the loop)
        auto run_box = [&](auto partial_tag, int bx, uint32_t w) {
            constexpr bool kPartial = decltype(partial_tag)::value;
            const uint32_t base = wrow + w * kWBox;
#pragma unroll
            for (int s = 0; s < SUB; ++s) {
                const int i = bx * SUB + s;                 // k-block within the segment
                if (!kPartial || i < nkb) {
                    const int lk = lk0 + i;                 // k-block within the CTA's slice (>= 0)
                    // this k-block's codes of the thread's two rows
                    uint32_t r0[2 * TW], r1[2 * TW];
                    if (TW == 2) {
                        const uint2 v0 = gemv_lds64(base + offs[s]);
                        const uint2 v1 = gemv_lds64(base + 1024 + offs[s]);
                        r0[0] = v0.x;
                        r0[1] = v0.y;
                        r1[0] = v1.x;
                        r1[1] = v1.y;
                    } else {
                        r0[0] = gemv_lds32(base + offs[s]);
                        r1[0] = gemv_lds32(base + 1024 + offs[s]);
                    }
                    if (s % GB == 0) {
                        // this group's constants from the table
                        const uint32_t ta = trow + static_cast<uint32_t>(lk) / GB * TE;
                        const uint32_t e0 = gemv_lds32(ta), e1 = gemv_lds32(ta + 8 * tstride * TE);
                        if (KIND != kCode4) {
                            sub0 = __byte_perm(e0, 0u, 0x1010);
                            sub1 = __byte_perm(e1, 0u, 0x1010);
                            sf0 = f16_bits_to_f32(static_cast<uint16_t>(e0 >> 16));
                            sf1 = f16_bits_to_f32(static_cast<uint16_t>(e1 >> 16));
                        } else {
                            sf0 = __uint_as_float(e0);
                            sf1 = __uint_as_float(e1);
                        }
                    }
                    // A fragments: 8 code pairs of each row as bf16x2
                    uint32_t f0[8], f1[8];
                    if (KIND == kInt4) {
                        int4_pairs(r0[0], mg, f0);
                        int4_pairs(r0[TW - 1], mg, f0 + 4);
                        int4_pairs(r1[0], mg, f1);
                        int4_pairs(r1[TW - 1], mg, f1 + 4);
                    } else if (KIND == kInt2) {
                        int2_pairs(r0[0], mg, f0);
                        int2_pairs(r1[0], mg, f1);
                    } else {
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            f0[q] = s_lut[__byte_perm(r0[0], 0u, 0x4440 + q)];
                            f0[4 + q] = s_lut[__byte_perm(r0[TW - 1], 0u, 0x4440 + q)];
                            f1[q] = s_lut[__byte_perm(r1[0], 0u, 0x4440 + q)];
                            f1[4 + q] = s_lut[__byte_perm(r1[TW - 1], 0u, 0x4440 + q)];
                        }
                    }
                    if (KIND != kCode4) {
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            f0[q] = sub_bf16x2(f0[q], sub0);
                            f1[q] = sub_bf16x2(f1[q], sub1);
                        }
                    }
                    // B fragments (permuted activations) and four MMA steps
                    const uint32_t xoff = static_cast<uint32_t>(lk) * 128;
                    uint2 bxf[4][NT8];
#pragma unroll
                    for (int tau = 0; tau < 4; ++tau)
#pragma unroll
                        for (int nt = 0; nt < NT8; ++nt)
                            bxf[tau][nt] = gemv_lds64(xthr[nt] + xoff + 8 * tau);
#pragma unroll
                    for (int tau = 0; tau < 4; ++tau)
#pragma unroll
                        for (int nt = 0; nt < NT8; ++nt) {
                            if (s % GB == 0 && tau < 2)
                                mma_m16n8k16_bf16_first(cg[tau & 1][nt], f0[2 * tau], f1[2 * tau], f0[2 * tau + 1],
                                                        f1[2 * tau + 1], bxf[tau][nt].x, bxf[tau][nt].y);
                            else
                                mma_m16n8k16_bf16(cg[tau & 1][nt], f0[2 * tau], f1[2 * tau], f0[2 * tau + 1],
                                                  f1[2 * tau + 1], bxf[tau][nt].x, bxf[tau][nt].y);
                        }
                    // end of a scale group: fold the group partial
                    if (s % GB == GB - 1) {
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
        };
        for (int bx = 0; bx < nbx; ++bx, ++c) {
            const uint32_t w = c % WS;
            if (!mbar_wait(&full[w], (c / WS) & 1u, s_abort)) break;
            if (bx < nfull)
                run_box(std::false_type{}, bx, w);
            else
                run_box(std::true_type{}, bx, w);
            // release the slot only after every loaded word has been used: an
            // arrive issued right behind the shared loads let the next TMA
            // write land before some of those loads had read the slot
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[w]);
        }
        if (KIND != kCode4 && far) {
            // groups stored with |zero| > 128 ran as (q - 0); add their
            // scale * (-zero) * (sum of x over the group) here
            for (int lg = lk0 / GB; lg < (lk0 + nkb) / GB; ++lg) {
                const int64_t gi = kb0 / GB + (lg - lk0 / GB);      // group within the row
                float k0 = 0.0f, k1 = 0.0f;
                if (ok0) {
                    const float z = f16_bits_to_f32(__ldg(p.zero + gr0 * p.ngroups + gi));
                    if (fabsf(z) > 128.0f) k0 = f16_bits_to_f32(__ldg(p.scale + gr0 * p.ngroups + gi)) * -z;
                }
                if (ok1) {
                    const float z = f16_bits_to_f32(__ldg(p.zero + gr1 * p.ngroups + gi));
                    if (fabsf(z) > 128.0f) k1 = f16_bits_to_f32(__ldg(p.scale + gr1 * p.ngroups + gi)) * -z;
                }
                if (k0 == 0.0f && k1 == 0.0f) continue;
#pragma unroll
                for (int nt = 0; nt < NT8; ++nt) {
                    const int tA = nt * 8 + 2 * j;
                    float sx0 = 0.0f, sx1 = 0.0f;
                    for (int kk = lg * GB * 64; kk < (lg + 1) * GB * 64; ++kk) {
                        if (tA < p.m) sx0 += bf16_bits_to_f32(sX[tA * xstride + kk]);
                        if (tA + 1 < p.m) sx1 += bf16_bits_to_f32(sX[(tA + 1) * xstride + kk]);
                    }
                    acc[nt][0] = fmaf(k0, sx0, acc[nt][0]);
                    acc[nt][1] = fmaf(k0, sx1, acc[nt][1]);
                    acc[nt][2] = fmaf(k1, sx0, acc[nt][2]);
                    acc[nt][3] = fmaf(k1, sx1, acc[nt][3]);
                }
            }
        }
        // -------------------------------------------------------------- segment epilogue
        auto lora = [&](int t, int oc) -> float {
            if (p.rank == 0) return 0.0f;
            float d = 0.0f;
            for (int u = 0; u < p.rank; ++u)
                d = fmaf(p.T[static_cast<int64_t>(t) * p.rank + u],
                         bf16_bits_to_f32(__ldg(p.B + static_cast<int64_t>(oc) * p.rank + u)), d);
            return p.s * d;
        };
        if (kb0 == 0 && nkb == p.kbt) {
            // this CTA covered the whole tile
#pragma unroll
            for (int nt = 0; nt < NT8; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int t = nt * 8 + 2 * j + (e & 1);
                    const bool ok = (e < 2) ? ok0 : ok1;
                    const int64_t r = (e < 2) ? gr0 : gr1;
                    if (ok && t < p.m) {
                        const int oc = p.perm ? p.perm[r] : static_cast<int>(r);
                        p.Y[static_cast<int64_t>(t) * p.ldy + oc] = acc[nt][e] + lora(t, oc);
                    }
                }
            continue;
        }
        // split tile.  Partial slot of (CTA b, tile t) is b + t: CTAs cover the
        // work in order, so no two (CTA, tile) pairs share a slot.
        const int cta_lo = static_cast<int>((static_cast<int64_t>(tile) * p.kbt) / p.share);
        const int cta_hi = static_cast<int>((static_cast<int64_t>(tile + 1) * p.kbt - 1) / p.share);
        if (kb0 + nkb < p.kbt) {
            // contributor (the tile's last k-block belongs to a later CTA)
            float* slot = p.partial + (static_cast<int64_t>(blockIdx.x) + tile) * p.m * 128;
#pragma unroll
            for (int nt = 0; nt < NT8; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int t = nt * 8 + 2 * j + (e & 1);
                    if (t < p.m) slot[t * 128 + rl0 + ((e < 2) ? 0 : 8)] = acc[nt][e];
                }
            asm volatile("bar.sync 1, 256;" ::: "memory");
            if (tid == 0) flag_publish(p.counters + tile);
            continue;
        }
        // this CTA finishes the tile: wait for the cta_hi - cta_lo contributors
        if (tid == 0) {
            if (!flag_wait_geq(p.counters + tile, static_cast<uint32_t>(cta_hi - cta_lo))) *s_abort = 1;
            p.counters[tile] = 0u;                     // left at zero for the next call
        }
        asm volatile("bar.sync 1, 256;" ::: "memory");
        // the contributors' partials in CTA order (QB CTAs' loads in flight
        // together), then this CTA's own sums
        constexpr int QB = NT8 == 1 ? 8 : 2;
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
                        part[q][nt][e] = (b0 + q < cta_hi && t < p.m)
                                             ? __ldcg(p.partial + ((static_cast<int64_t>(b0 + q) + tile) * p.m + t) * 128 +
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
                if (ok && t < p.m) {
                    const int oc = p.perm ? p.perm[r] : static_cast<int>(r);
                    p.Y[static_cast<int64_t>(t) * p.ldy + oc] = (v[nt][e] + acc[nt][e]) + lora(t, oc);
                }
            }
    }
}

}  // namespace lbq
