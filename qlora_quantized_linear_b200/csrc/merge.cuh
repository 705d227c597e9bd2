// merge.cuh -- merging a low-rank adapter into the weight, and removing it
// again (GreenBit article, introduction: after QLoRA fine-tuning the LoRA
// module is merged into the full-precision model).
//
//   merge:    W_out[i, j] = bf16(W_hat[i, j] + s * sum_u B[i, u] A[u, j])
//   unmerge:  W_out[i, j] = bf16(W[i, j]     - s * sum_u B[i, u] A[u, j])
//
// Every element is evaluated in binary32 in one fixed order: d = fma(B, A, d)
// over u = 0 .. r-1, t = s * d, v = W +/- t, then bf16 round-to-nearest-even.
// One order on every path makes a merged weight, and so its re-quantization,
// reproducible bit for bit.
//
// Bound by HBM (the bf16 output is 2 bytes per weight against 0.5 read for
// INT4; the adapter stays in L2).  A CTA owns a 64-row x 128-column tile, a
// thread 8 rows x 4 consecutive columns, with the 32 partial sums in
// registers.  The thread's weight words go out first; meanwhile the adapter
// is staged in shared memory as fp32 (A as 16-byte loads along the columns, B
// as 16-byte loads along each row when the rank is a multiple of 8), so that
// one 16-byte load of A and two broadcast loads of B feed 16 packed fp32 FMAs
// (fma.rn.f32x2 on pairs of rows).
#pragma once

#include "quantize.cuh"

namespace lbq {

constexpr int kMergeThreads = 256;
constexpr int kMergeRows = 64;          // rows per CTA tile (8 per warp)
constexpr int kMergeCols = 128;         // columns per CTA tile (4 per lane)
constexpr int kMergeRankChunk = 32;     // adapter terms staged at a time

enum { kMergeInt4 = 0, kMergeInt2 = 1, kMergeCode4 = 2, kMergeBf16 = 3 };

struct MergeParams {
    int n, k;
    int ngroups;                  // MinMax: k / group
    const uint8_t* packed;
    const uint16_t* scale;
    const uint16_t* zero;
    const float* absmax;          // codebook without double quant
    const int8_t* q8;             // codebook with double quant
    const float* s2;
    const float* offset;
    const float* codebook;
    const uint16_t* W;            // unmerge: bf16 [n, k]
    const uint16_t* A;            // bf16 [rank, k]
    const uint16_t* B;            // bf16 [n, rank]
    int rank;
    float s;
    uint16_t* out;                // bf16 [n, k]
};

__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) { return pack_bf16x2_rn(lo, hi); }

// Two fp32 values in one 64-bit register pair, for the packed fp32 FMA.
__device__ __forceinline__ uint64_t pack_f32x2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ void unpack_f32x2(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

// d = fma(a, b, d) on both halves: two IEEE fused multiply-adds in one
// instruction, each rounded once exactly as fmaf.
__device__ __forceinline__ void fma_x2(uint64_t& d, uint64_t a, uint64_t b) {
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(d) : "l"(a), "l"(b));
}

// The weight inputs of one thread for one row tile (loaded a tile ahead).
struct MergeIn {
    uint32_t raw[8];              // packed codes of the 8 rows (or bf16 pairs x)
    uint32_t raw2[8];             // bf16 pairs y (removal)
    uint32_t aux[8];              // MinMax: fp16 zero | fp16 scale << 16; codebook: fp32 absmax bits
};

template <int MODE>
__device__ __forceinline__ void merge_load(const MergeParams& p, int64_t row0, int col0, MergeIn& in) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t row = row0 + i;
        in.raw[i] = in.raw2[i] = in.aux[i] = 0u;
        if (row >= p.n || col0 >= p.k) continue;
        const int64_t e0 = row * p.k + col0;                  // first element
        if (MODE == kMergeInt4 || MODE == kMergeCode4) {
            in.raw[i] = __ldg(reinterpret_cast<const uint16_t*>(p.packed) + e0 / 4);
        } else if (MODE == kMergeInt2) {
            in.raw[i] = __ldg(p.packed + e0 / 4);
        } else {
            const uint2 w = __ldg(reinterpret_cast<const uint2*>(p.W + e0));
            in.raw[i] = w.x;
            in.raw2[i] = w.y;
        }
        if (MODE == kMergeInt4 || MODE == kMergeInt2) {
            const int64_t g = row * p.ngroups + col0 / (p.k / p.ngroups);
            in.aux[i] = static_cast<uint32_t>(__ldg(p.zero + g)) | (static_cast<uint32_t>(__ldg(p.scale + g)) << 16);
        } else if (MODE == kMergeCode4) {
            const int64_t b = e0 / 64;
            in.aux[i] = __float_as_uint((p.q8 != nullptr) ? double_dequant(p.q8[b], p.s2[b >> 8], *p.offset)
                                                          : __ldg(p.absmax + b));
        }
    }
}

// MODE: the source of the weight (kMerge*); a removal reads a bf16 weight and
// subtracts, every other mode dequantizes and adds.
template <int MODE>
__global__ void __launch_bounds__(kMergeThreads, 3) lora_merge_kernel(const MergeParams p) {
    __shared__ __align__(16) float sA[kMergeRankChunk][kMergeCols];     // 16 KB
    __shared__ __align__(16) float sB[kMergeRankChunk][kMergeRows];     // 8 KB
    __shared__ float s_cb[16];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t tile_row = static_cast<int64_t>(blockIdx.y) * kMergeRows;
    const int tile_col = blockIdx.x * kMergeCols;
    const int col0 = tile_col + lane * 4;                     // this thread's 4 columns
    const int64_t row0 = tile_row + warp * 8;                 // and 8 rows
    if (MODE == kMergeCode4 && tid < 16) s_cb[tid] = p.codebook[tid];

    // the weight words of the thread's 8 rows go out first
    MergeIn in;
    merge_load<MODE>(p, row0, col0, in);

    // the partial sums as pairs of rows (2 ip, 2 ip + 1) per column c, so that
    // the B values of two rows (adjacent in shared memory) form one operand and
    // only the A value of a column is duplicated into a pair
    uint64_t dp[4][4];
#pragma unroll
    for (int ip = 0; ip < 4; ++ip)
#pragma unroll
        for (int c = 0; c < 4; ++c) dp[ip][c] = 0ull;

    for (int u0 = 0; u0 < p.rank; u0 += kMergeRankChunk) {
        const int ur = min(kMergeRankChunk, p.rank - u0);
        if (u0 > 0) __syncthreads();                          // the previous chunk is consumed
        // A[u0 + u][tile columns] as fp32, 8 columns (16 bytes of bf16) per step
        for (int e = tid; e < ur * (kMergeCols / 8); e += kMergeThreads) {
            const int u = e / (kMergeCols / 8), c8 = e - u * (kMergeCols / 8);
            const int col = tile_col + c8 * 8;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (col < p.k) v = __ldg(reinterpret_cast<const uint4*>(p.A + static_cast<int64_t>(u0 + u) * p.k + col));
            float4* dst = reinterpret_cast<float4*>(&sA[u][c8 * 8]);
            dst[0] = make_float4(bf16_bits_to_f32(v.x & 0xFFFFu), bf16_bits_to_f32(v.x >> 16),
                                 bf16_bits_to_f32(v.y & 0xFFFFu), bf16_bits_to_f32(v.y >> 16));
            dst[1] = make_float4(bf16_bits_to_f32(v.z & 0xFFFFu), bf16_bits_to_f32(v.z >> 16),
                                 bf16_bits_to_f32(v.w & 0xFFFFu), bf16_bits_to_f32(v.w >> 16));
        }
        // B[tile rows][u0 + u] transposed to [u][row]
        if ((p.rank & 7) == 0) {
            // 8 rank terms of one row (16 bytes) per step: rows are contiguous in B
            const int pieces = ur / 8;
            for (int e = tid; e < kMergeRows * pieces; e += kMergeThreads) {
                const int rr = e / pieces, pc = e - rr * pieces;
                const int64_t row = tile_row + rr;
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (row < p.n) v = __ldg(reinterpret_cast<const uint4*>(p.B + row * p.rank + u0 + pc * 8));
                const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    sB[pc * 8 + 2 * h][rr] = bf16_bits_to_f32(w4[h] & 0xFFFFu);
                    sB[pc * 8 + 2 * h + 1][rr] = bf16_bits_to_f32(w4[h] >> 16);
                }
            }
        } else {
            for (int e = tid; e < ur * kMergeRows; e += kMergeThreads) {
                const int u = e / kMergeRows, rr = e - u * kMergeRows;
                const int64_t row = tile_row + rr;
                sB[u][rr] = row < p.n ? bf16_bits_to_f32(__ldg(p.B + row * p.rank + u0 + u)) : 0.0f;
            }
        }
        __syncthreads();
        for (int u = 0; u < ur; ++u) {
            const float4 a = *reinterpret_cast<const float4*>(&sA[u][lane * 4]);
            const float4 b0 = *reinterpret_cast<const float4*>(&sB[u][warp * 8]);
            const float4 b1 = *reinterpret_cast<const float4*>(&sB[u][warp * 8 + 4]);
            const uint64_t bp[4] = {pack_f32x2(b0.x, b0.y), pack_f32x2(b0.z, b0.w), pack_f32x2(b1.x, b1.y),
                                    pack_f32x2(b1.z, b1.w)};
            const uint64_t ap[4] = {pack_f32x2(a.x, a.x), pack_f32x2(a.y, a.y), pack_f32x2(a.z, a.z),
                                    pack_f32x2(a.w, a.w)};
#pragma unroll
            for (int ip = 0; ip < 4; ++ip)
#pragma unroll
                for (int c = 0; c < 4; ++c) fma_x2(dp[ip][c], bp[ip], ap[c]);
        }
    }
    if (MODE == kMergeCode4 && p.rank == 0) __syncthreads();  // the codebook copy (else done by the chunk barrier)
    if (col0 >= p.k) return;                                  // k % 8 == 0: a thread's 4 columns are all in or out
    float d[8][4];
#pragma unroll
    for (int ip = 0; ip < 4; ++ip)
#pragma unroll
        for (int c = 0; c < 4; ++c) unpack_f32x2(dp[ip][c], d[2 * ip][c], d[2 * ip + 1][c]);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t row = row0 + i;
        if (row >= p.n) continue;
        float w[4];
        if (MODE == kMergeInt4 || MODE == kMergeCode4) {
            // bytes (c0 << 4 | c1), (c2 << 4 | c3): the first code in the high nibble
            const uint32_t r = in.raw[i];
            const uint32_t q[4] = {(r >> 4) & 15u, r & 15u, (r >> 12) & 15u, (r >> 8) & 15u};
            const float zf = f16_bits_to_f32(static_cast<uint16_t>(in.aux[i] & 0xFFFFu));
            const float sf = f16_bits_to_f32(static_cast<uint16_t>(in.aux[i] >> 16));
#pragma unroll
            for (int c = 0; c < 4; ++c)
                w[c] = (MODE == kMergeInt4) ? __fmul_rn(__fsub_rn(static_cast<float>(q[c]), zf), sf)
                                            : __fmul_rn(s_cb[q[c]], __uint_as_float(in.aux[i]));
        } else if (MODE == kMergeInt2) {
            const float zf = f16_bits_to_f32(static_cast<uint16_t>(in.aux[i] & 0xFFFFu));
            const float sf = f16_bits_to_f32(static_cast<uint16_t>(in.aux[i] >> 16));
#pragma unroll
            for (int c = 0; c < 4; ++c)
                w[c] = __fmul_rn(__fsub_rn(static_cast<float>((in.raw[i] >> (6 - 2 * c)) & 3u), zf), sf);
        } else {
            w[0] = bf16_bits_to_f32(in.raw[i] & 0xFFFFu);
            w[1] = bf16_bits_to_f32(in.raw[i] >> 16);
            w[2] = bf16_bits_to_f32(in.raw2[i] & 0xFFFFu);
            w[3] = bf16_bits_to_f32(in.raw2[i] >> 16);
        }
        float v[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const float t = __fmul_rn(p.s, d[i][c]);
            v[c] = (MODE == kMergeBf16) ? __fsub_rn(w[c], t) : __fadd_rn(w[c], t);
        }
        *reinterpret_cast<uint2*>(p.out + row * p.k + col0) = make_uint2(bf16x2_rn(v[0], v[1]), bf16x2_rn(v[2], v[3]));
    }
}

}  // namespace lbq
