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
// INT4; the adapter stays in L2): a CTA owns a 64-row x 128-column tile, each
// thread 8 rows x 4 consecutive columns.  The 32 partial sums stay in
// registers; the adapter is staged in shared memory as fp32 in rank chunks of
// 32, one 16-byte load of A and two broadcast loads of B feeding 32 FMAs.
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

// MODE: the source of the weight (kMerge*); unmerge reads a bf16 weight and
// subtracts, every other mode dequantizes and adds.
template <int MODE>
__global__ void __launch_bounds__(kMergeThreads) lora_merge_kernel(const MergeParams p) {
    __shared__ __align__(16) float sA[kMergeRankChunk][kMergeCols];     // 16 KB
    __shared__ __align__(16) float sB[kMergeRankChunk][kMergeRows];     // 8 KB
    __shared__ float s_cb[16];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t tile_row = static_cast<int64_t>(blockIdx.y) * kMergeRows;
    const int tile_col = blockIdx.x * kMergeCols;
    const int col0 = tile_col + lane * 4;                     // this thread's 4 columns
    const int64_t row0 = tile_row + warp * 8;                 // and 8 rows
    if (MODE == kMergeCode4 && tid < 16) s_cb[tid] = p.codebook[tid];

    float d[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int c = 0; c < 4; ++c) d[i][c] = 0.0f;

    for (int u0 = 0; u0 < p.rank; u0 += kMergeRankChunk) {
        const int ur = min(kMergeRankChunk, p.rank - u0);
        __syncthreads();                                      // the previous chunk is consumed
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
        // B[tile rows][u0 + u], transposed to [u][row] (consecutive lanes take
        // consecutive rows, so the shared stores do not conflict)
        for (int e = tid; e < ur * kMergeRows; e += kMergeThreads) {
            const int u = e / kMergeRows, rr = e - u * kMergeRows;
            const int64_t row = tile_row + rr;
            sB[u][rr] = row < p.n ? bf16_bits_to_f32(__ldg(p.B + row * p.rank + u0 + u)) : 0.0f;
        }
        __syncthreads();
        for (int u = 0; u < ur; ++u) {
            const float4 a = *reinterpret_cast<const float4*>(&sA[u][lane * 4]);
            const float4 b0 = *reinterpret_cast<const float4*>(&sB[u][warp * 8]);
            const float4 b1 = *reinterpret_cast<const float4*>(&sB[u][warp * 8 + 4]);
            const float av[4] = {a.x, a.y, a.z, a.w};
            const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int c = 0; c < 4; ++c) d[i][c] = fmaf(bv[i], av[c], d[i][c]);
        }
    }
    if (MODE == kMergeCode4 && p.rank == 0) __syncthreads();  // the codebook copy (else done by the chunk barriers)
    if (col0 >= p.k) return;                                  // k % 8 == 0: a thread's 4 columns are all in or out

    // the weight: all eight rows' loads first, then the arithmetic
    uint32_t raw[8];
    float amax[8], zf[8], sf[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t row = row0 + i;
        raw[i] = 0u;
        amax[i] = zf[i] = sf[i] = 0.0f;
        if (row >= p.n) continue;
        const int64_t e0 = row * p.k + col0;                  // first element
        if (MODE == kMergeInt4 || MODE == kMergeCode4) {
            raw[i] = __ldg(reinterpret_cast<const uint16_t*>(p.packed) + e0 / 4);
        } else if (MODE == kMergeInt2) {
            raw[i] = __ldg(p.packed + e0 / 4);
        }
        if (MODE == kMergeInt4 || MODE == kMergeInt2) {
            const int64_t g = row * p.ngroups + col0 / (p.k / p.ngroups);
            zf[i] = f16_bits_to_f32(__ldg(p.zero + g));
            sf[i] = f16_bits_to_f32(__ldg(p.scale + g));
        } else if (MODE == kMergeCode4) {
            const int64_t b = e0 / 64;
            amax[i] = (p.q8 != nullptr) ? double_dequant(p.q8[b], p.s2[b >> 8], *p.offset) : __ldg(p.absmax + b);
        }
    }
    uint2 wb[8];
    if (MODE == kMergeBf16) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int64_t row = row0 + i;
            wb[i] = row < p.n ? __ldg(reinterpret_cast<const uint2*>(p.W + row * p.k + col0)) : make_uint2(0u, 0u);
        }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t row = row0 + i;
        if (row >= p.n) continue;
        float w[4];
        if (MODE == kMergeInt4 || MODE == kMergeCode4) {
            // bytes (c0 << 4 | c1), (c2 << 4 | c3): the first code in the high nibble
            const uint32_t q[4] = {(raw[i] >> 4) & 15u, raw[i] & 15u, (raw[i] >> 12) & 15u, (raw[i] >> 8) & 15u};
#pragma unroll
            for (int c = 0; c < 4; ++c)
                w[c] = (MODE == kMergeInt4) ? __fmul_rn(__fsub_rn(static_cast<float>(q[c]), zf[i]), sf[i])
                                            : __fmul_rn(s_cb[q[c]], amax[i]);
        } else if (MODE == kMergeInt2) {
#pragma unroll
            for (int c = 0; c < 4; ++c)
                w[c] = __fmul_rn(__fsub_rn(static_cast<float>((raw[i] >> (6 - 2 * c)) & 3u), zf[i]), sf[i]);
        } else {
            w[0] = bf16_bits_to_f32(wb[i].x & 0xFFFFu);
            w[1] = bf16_bits_to_f32(wb[i].x >> 16);
            w[2] = bf16_bits_to_f32(wb[i].y & 0xFFFFu);
            w[3] = bf16_bits_to_f32(wb[i].y >> 16);
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
