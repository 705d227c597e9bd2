// select.cuh -- choosing the INT4 channels of a channel-mix weight by their
// sensitivity to quantization (GreenBit.AI article, 模型量化 (1): the bit width
// of each output channel follows how much quantizing it to fewer bits costs).
//
//   m2[k]    = (1/T) sum_t x[t,k]^2                     calibration activations
//   e4, e2   = W_hat - w of the MinMax INT4 g128 / INT2 g64 quantization
//   score[c] = sum_k m2[k] * (e2[c,k]^2 - e4[c,k]^2)
//
// score[c] is the rise of the expected squared output error of channel c when
// it goes from INT4 to INT2 (second moments on the diagonal).  The n4 channels
// with the highest score become INT4 (the lower channel first among equal
// scores); perm lists them in ascending order, then the other channels.
//
// Kernels: the second moments (one thread per input feature, fp64, the tokens
// in order); the scores (one warp per channel, the same exact MinMax
// arithmetic as the quantize kernels, fp64 sums); the ranks (one thread per
// channel, counting the channels that come before it); the permutation (one
// CTA, a scan of the selection flags).
#pragma once

#include "quantize.cuh"

namespace lbq {

__global__ void __launch_bounds__(256) second_moment_kernel(const uint16_t* __restrict__ X, int64_t t, int64_t k,
                                                            double* __restrict__ m2) {
    const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (j >= k) return;
    double acc = 0.0;
    for (int64_t i = 0; i < t; ++i) {
        const double x = static_cast<double>(bf16_bits_to_f32(__ldg(X + i * k + j)));
        acc = __dadd_rn(acc, __dmul_rn(x, x));
    }
    m2[j] = __ddiv_rn(acc, static_cast<double>(t));
}

// The MinMax round trip W_hat of a lane's 8 consecutive elements, its group
// being GROUP / 8 consecutive lanes (all 32 lanes take part in the shuffles):
// the arithmetic of minmax_quantize_kernel, then W_hat = (code - zero) * scale
// as one fp32 product.
template <int BITS>
__device__ __forceinline__ void minmax_roundtrip8(const float (&v)[8], float (&wh)[8]) {
    constexpr int GROUP = (BITS == 4) ? 128 : 64;
    constexpr int LPG = GROUP / 8;
    constexpr float Q = static_cast<float>((1 << BITS) - 1);
    float mn = v[0], mx = v[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) {
        mn = fminf(mn, v[i]);
        mx = fmaxf(mx, v[i]);
    }
#pragma unroll
    for (int off = LPG / 2; off > 0; off >>= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, off));
        mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
    }
    mn = __fadd_rn(mn, 0.0f);
    mx = __fadd_rn(mx, 0.0f);
    const float r = __fsub_rn(mx, mn);
    uint16_t s16 = f32_to_f16_bits(__fdiv_rn(r, Q));
    if (r == 0.0f || (s16 & 0x7FFFu) == 0) s16 = 0x3C00u;  // 1.0
    const float sf = f16_bits_to_f32(s16);
    const float zf = f16_bits_to_f32(f32_to_f16_bits(rintf(__fdiv_rn(-mn, sf))));
    const float rs = __frcp_rn(sf);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float q = __fadd_rn(rint_div(v[i], sf, rs), zf);
        q = fminf(fmaxf(q, 0.0f), Q);
        wh[i] = __fmul_rn(__fsub_rn(q, zf), sf);
    }
}

// One warp per channel; the row is walked 256 elements (32 lanes x 8) at a
// time, whole INT4 and INT2 groups per step.  k % 128 == 0.
__global__ void __launch_bounds__(256) channel_score_kernel(const uint16_t* __restrict__ W, int64_t n, int64_t k,
                                                            const double* __restrict__ m2,
                                                            double* __restrict__ score) {
    const int lane = threadIdx.x & 31;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (row >= n) return;                                  // whole warps
    const uint4* w4 = reinterpret_cast<const uint4*>(W + row * k);
    double sc = 0.0;
    for (int64_t base = 0; base < k; base += 256) {
        const int64_t col = base + 8 * lane;
        const bool valid = col < k;                        // whole 128-element groups
        const uint4 raw = valid ? __ldg(w4 + (col >> 3)) : make_uint4(0, 0, 0, 0);
        const uint32_t words[4] = {raw.x, raw.y, raw.z, raw.w};
        float v[8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[2 * i] = bf16_bits_to_f32(words[i] & 0xFFFFu);
            v[2 * i + 1] = bf16_bits_to_f32(words[i] >> 16);
        }
        float w4h[8], w2h[8];
        minmax_roundtrip8<4>(v, w4h);
        minmax_roundtrip8<2>(v, w2h);
        if (!valid) continue;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const double w = static_cast<double>(v[i]);
            const double e4 = __dsub_rn(static_cast<double>(w4h[i]), w);
            const double e2 = __dsub_rn(static_cast<double>(w2h[i]), w);
            sc = __dadd_rn(sc, __dmul_rn(__ldg(m2 + col + i), __dsub_rn(__dmul_rn(e2, e2), __dmul_rn(e4, e4))));
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sc = __dadd_rn(sc, __shfl_xor_sync(0xFFFFFFFFu, sc, off));
    if (lane == 0) score[row] = sc;
}

// sel[c] = 1 when fewer than n4 channels come before c (a higher score, or
// an equal score and a lower index).
__global__ void __launch_bounds__(256) channel_rank_kernel(const double* __restrict__ score, int64_t n, int64_t n4,
                                                           uint8_t* __restrict__ sel) {
    __shared__ double s_tile[2048];
    const int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const double sc = c < n ? score[c] : 0.0;
    int64_t rank = 0;
    for (int64_t d0 = 0; d0 < n; d0 += 2048) {
        const int cnt = static_cast<int>(n - d0 < 2048 ? n - d0 : 2048);
        __syncthreads();
        for (int i = threadIdx.x; i < cnt; i += blockDim.x) s_tile[i] = score[d0 + i];
        __syncthreads();
        for (int i = 0; i < cnt; ++i) {
            const double sd = s_tile[i];
            rank += (sd > sc || (sd == sc && d0 + i < c)) ? 1 : 0;
        }
    }
    if (c < n) sel[c] = rank < n4 ? 1 : 0;
}

// One CTA of 1024 threads: perm[position] = c, the selected channels first in
// ascending order, then the others.
__global__ void __launch_bounds__(1024) channel_perm_kernel(const uint8_t* __restrict__ sel, int64_t n, int64_t n4,
                                                            int32_t* __restrict__ perm) {
    __shared__ int s_warp[32];
    __shared__ int64_t s_carry;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid == 0) s_carry = 0;
    __syncthreads();
    for (int64_t base = 0; base < n; base += 1024) {
        const int64_t c = base + tid;
        const int f = (c < n) ? sel[c] : 0;
        // inclusive scan of the flags within the chunk
        int x = f;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xFFFFFFFFu, x, off);
            if (lane >= off) x += y;
        }
        if (lane == 31) s_warp[warp] = x;
        __syncthreads();
        if (warp == 0) {
            int w = s_warp[lane];
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int y = __shfl_up_sync(0xFFFFFFFFu, w, off);
                if (lane >= off) w += y;
            }
            s_warp[lane] = w;
        }
        __syncthreads();
        const int64_t before = s_carry + (warp > 0 ? s_warp[warp - 1] : 0) + (x - f);   // selected before c
        if (c < n) perm[f ? before : n4 + (c - before)] = static_cast<int32_t>(c);
        __syncthreads();
        if (tid == 1023) s_carry += s_warp[31];
        __syncthreads();
    }
}

// out[i, :] = W[rows[i], :] (bf16 rows, 16 bytes per thread).
__global__ void __launch_bounds__(256) gather_rows_kernel(const uint4* __restrict__ W, int64_t k8,
                                                          const int32_t* __restrict__ rows, int64_t count,
                                                          uint4* __restrict__ out) {
    const int64_t total = count * k8;
    for (int64_t e = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; e < total;
         e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t i = e / k8, j = e - i * k8;
        out[e] = __ldg(W + static_cast<int64_t>(rows[i]) * k8 + j);
    }
}

}  // namespace lbq
