// lora.cuh -- low-rank adapter side products (QLoRA explainer, section
// QLoRA技术原理: only the adapters A, B are trained; gradients pass through the
// frozen quantized weight).
//
//   T  = X A^T      [m, r]   row reduction over k      (lora_rowdot_kernel)
//   U  = dY B       [m, r]   row reduction over n      (lora_rowdot_kernel)
//   dA = s U^T X    [r, k]   reduction over the m rows (lora_colgrad_kernel)
//   dB = s dY^T T   [n, r]   reduction over the m rows (lora_colgrad_kernel)
//
// These are skinny (r <= 64) and bandwidth-bound: each streams its bf16 input
// once with 16-byte loads and keeps the rank dimension in registers.  All
// accumulation is fp32 in a fixed order, so results are deterministic.
#pragma once

#include "common.cuh"

namespace lbq {

constexpr int kLoraMaxRank = 64;

// out[row, t] = sum_c in[row, c] * P(t, c),  t < r,
// where P(t, c) = wt[t * ldw + c]     (T = X A^T: wt = A [r, k], "row" layout)
//    or P(t, c) = wt[c * r + t]       (U = dY B:  wt = B [n, r], "col" layout).
// One CTA per row; 256 threads split the reduction in chunks of 8.
template <bool kColLayout>
__global__ void __launch_bounds__(256) lora_rowdot_kernel(const uint16_t* __restrict__ in, int64_t len,
                                                          const uint16_t* __restrict__ wt, int r,
                                                          float* __restrict__ out) {
    __shared__ float s_part[8][kLoraMaxRank];
    const int64_t row = blockIdx.x;
    const uint4* x4 = reinterpret_cast<const uint4*>(in + row * len);
    const int64_t nch = len / 8;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int t0 = 0; t0 < r; t0 += 16) {
        float acc[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) acc[t] = 0.0f;
        for (int64_t ch = threadIdx.x; ch < nch; ch += blockDim.x) {
            const uint4 xr = __ldg(x4 + ch);
            const uint32_t xw[4] = {xr.x, xr.y, xr.z, xr.w};
            float xv[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                xv[2 * i] = bf16_bits_to_f32(xw[i] & 0xFFFFu);
                xv[2 * i + 1] = bf16_bits_to_f32(xw[i] >> 16);
            }
            if (!kColLayout) {
#pragma unroll
                for (int t = 0; t < 16; ++t) {
                    if (t0 + t < r) {
                        const uint4 ar = __ldg(reinterpret_cast<const uint4*>(wt + (t0 + t) * len) + ch);
                        const uint32_t aw[4] = {ar.x, ar.y, ar.z, ar.w};
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            acc[t] = fmaf(xv[2 * i], bf16_bits_to_f32(aw[i] & 0xFFFFu), acc[t]);
                            acc[t] = fmaf(xv[2 * i + 1], bf16_bits_to_f32(aw[i] >> 16), acc[t]);
                        }
                    }
                }
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint16_t* brow = wt + (ch * 8 + i) * r + t0;
#pragma unroll
                    for (int t = 0; t < 16; ++t)
                        if (t0 + t < r) acc[t] = fmaf(xv[i], bf16_bits_to_f32(__ldg(brow + t)), acc[t]);
                }
            }
        }
#pragma unroll
        for (int t = 0; t < 16; ++t) {
            float v = acc[t];
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
            if (lane == 0 && t0 + t < r) s_part[warp][t0 + t] = v;
        }
    }
    __syncthreads();
    if (threadIdx.x < r) {
        float v = 0.0f;
#pragma unroll
        for (int w = 0; w < 8; ++w) v += s_part[w][threadIdx.x];
        out[row * r + threadIdx.x] = v;
    }
}

// grad[c, t] = s * sum_i in[i, c] * coef[i, t]   for c in a tile of 32 columns,
// written to grad[c * ocs + t * ots]:
//   dA: in = X [m, k],  coef = U [m, r], ocs = 1, ots = k
//   dB: in = dY [m, n], coef = T [m, r], ocs = r, ots = 1
// 256 threads: 32 columns x 8 rank groups; rows are staged through shared
// memory 64 at a time with 16-byte loads.
__global__ void __launch_bounds__(256) lora_colgrad_kernel(const uint16_t* __restrict__ in, int64_t m,
                                                           int64_t ncols, const float* __restrict__ coef, int r,
                                                           float s, float* __restrict__ grad, int64_t ocs,
                                                           int64_t ots) {
    constexpr int CT = 32, MC = 64;
    __shared__ float s_in[MC][CT + 1];
    __shared__ float s_coef[MC][kLoraMaxRank];
    const int64_t c0 = static_cast<int64_t>(blockIdx.x) * CT;
    const int cl = threadIdx.x & 31;  // column within the tile
    const int tg = threadIdx.x >> 5;  // rank group: t = tg, tg + 8, ...
    float acc[kLoraMaxRank / 8];
#pragma unroll
    for (int j = 0; j < kLoraMaxRank / 8; ++j) acc[j] = 0.0f;
    for (int64_t i0 = 0; i0 < m; i0 += MC) {
        const int rows = static_cast<int>((m - i0) < MC ? (m - i0) : MC);
        // stage MC x 32 bf16 of `in` (4 x 16-byte chunks per row)
        for (int e = threadIdx.x; e < MC * 4; e += blockDim.x) {
            const int rr = e >> 2, q = e & 3;
            float v[8] = {0, 0, 0, 0, 0, 0, 0, 0};
            const int64_t col = c0 + q * 8;
            if (rr < rows && col < ncols) {
                const uint4 raw = __ldg(reinterpret_cast<const uint4*>(in + (i0 + rr) * ncols + col));
                const uint32_t w4[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    v[2 * i] = bf16_bits_to_f32(w4[i] & 0xFFFFu);
                    v[2 * i + 1] = bf16_bits_to_f32(w4[i] >> 16);
                }
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) s_in[rr][q * 8 + i] = v[i];
        }
        for (int e = threadIdx.x; e < MC * r; e += blockDim.x) {
            const int rr = e / r, t = e - rr * r;
            s_coef[rr][t] = (rr < rows) ? coef[(i0 + rr) * r + t] : 0.0f;
        }
        __syncthreads();
        for (int rr = 0; rr < rows; ++rr) {
            const float x = s_in[rr][cl];
#pragma unroll
            for (int j = 0; j < kLoraMaxRank / 8; ++j) {
                const int t = tg + 8 * j;
                if (t < r) acc[j] = fmaf(x, s_coef[rr][t], acc[j]);
            }
        }
        __syncthreads();
    }
    const int64_t c = c0 + cl;
    if (c < ncols) {
#pragma unroll
        for (int j = 0; j < kLoraMaxRank / 8; ++j) {
            const int t = tg + 8 * j;
            if (t < r) grad[c * ocs + t * ots] = __fmul_rn(s, acc[j]);
        }
    }
}

}  // namespace lbq
