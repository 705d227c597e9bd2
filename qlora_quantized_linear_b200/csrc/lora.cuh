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
// once with 16-byte loads.  For more than a few rows they run on register
// tensor-core MMAs (mma.sync m16n8k16, bf16 in, fp32 accumulate); for decode
// sizes the one-CTA-per-row reduction below is used.  All accumulation is in
// a fixed order, so results are deterministic.
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

// ---------------------------------------------------------------------------
// tensor-core versions
// ---------------------------------------------------------------------------
__device__ __forceinline__ void lora_mma(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// out[row, t] = sum_c in[row, c] * W(c, t), t < r <= 8 * R8, with
//   W(c, t) = wt[t * len + c]   (T = X A^T: wt = A [r, len], row layout)
//   W(c, t) = wt[c * r + t]     (U = dY B:  wt = B [len, r], col layout).
// A CTA owns 16 rows; its 8 warps take every 8th 32-wide step of the
// reduction.  Lane (g, j) loads 8 consecutive elements of rows g and g + 8
// and of column g of W: the MMA's k order is permuted the same way on both
// sides (virtual k 2j, 2j+1 / 2j+8, 2j+9 hold actual elements 8j .. 8j+3 in
// the first MMA and 8j+4 .. 8j+7 in the second).  The warps' partials are
// summed in warp order in shared memory.  len % 8 == 0.
template <bool kCol, int R8>
__global__ void __launch_bounds__(256) lora_rows_mma_kernel(const uint16_t* __restrict__ in, int64_t m, int64_t len,
                                                            const uint16_t* __restrict__ wt, int r,
                                                            float* __restrict__ out) {
    __shared__ float s_red[8][16][8 * R8 + 1];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, j = lane & 3;
    const int64_t row0 = static_cast<int64_t>(blockIdx.x) * 16;
    const int64_t ra = row0 + g, rb = ra + 8;
    const uint16_t* pa = in + (ra < m ? ra : 0) * len;
    const uint16_t* pb = in + (rb < m ? rb : 0) * len;
    const bool oka = ra < m, okb = rb < m;
    float acc[R8][4];
#pragma unroll
    for (int nt = 0; nt < R8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[nt][e] = 0.0f;
    const int64_t nstep = (len + 31) / 32;
    for (int64_t st = warp; st < nstep; st += 8) {
        const int64_t k0 = st * 32 + 8 * j;
        const bool kin = k0 < len;                 // len % 8 == 0: all 8 or none
        const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
        const uint4 xa = (kin && oka) ? __ldg(reinterpret_cast<const uint4*>(pa + k0)) : z4;
        const uint4 xb = (kin && okb) ? __ldg(reinterpret_cast<const uint4*>(pb + k0)) : z4;
#pragma unroll
        for (int nt = 0; nt < R8; ++nt) {
            const int t = nt * 8 + g;
            uint32_t b[4] = {0u, 0u, 0u, 0u};
            if (kin && t < r) {
                if (!kCol) {
                    const uint4 w4 = __ldg(reinterpret_cast<const uint4*>(wt + static_cast<int64_t>(t) * len + k0));
                    b[0] = w4.x;
                    b[1] = w4.y;
                    b[2] = w4.z;
                    b[3] = w4.w;
                } else {
                    const uint16_t* wc = wt + k0 * r + t;
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        b[q] = static_cast<uint32_t>(__ldg(wc + (2 * q) * r)) |
                               (static_cast<uint32_t>(__ldg(wc + (2 * q + 1) * r)) << 16);
                }
            }
            lora_mma(acc[nt], xa.x, xb.x, xa.y, xb.y, b[0], b[1]);
            lora_mma(acc[nt], xa.z, xb.z, xa.w, xb.w, b[2], b[3]);
        }
    }
#pragma unroll
    for (int nt = 0; nt < R8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) s_red[warp][g + 8 * (e >> 1)][nt * 8 + 2 * j + (e & 1)] = acc[nt][e];
    __syncthreads();
    for (int e = threadIdx.x; e < 16 * 8 * R8; e += blockDim.x) {
        const int rr = e / (8 * R8), t = e - rr * (8 * R8);
        if (t < r && row0 + rr < m) {
            float v = 0.0f;
#pragma unroll
            for (int w = 0; w < 8; ++w) v += s_red[w][rr][t];
            out[(row0 + rr) * r + t] = v;
        }
    }
}

// grad(c, t) = s * sum_i in[i, c] * coef[i, t], written to grad[c * ocs + t * ots]:
//   dA: in = X [m, k],  coef = U [m, r], ocs = 1, ots = k
//   dB: in = dY [m, n], coef = T [m, r], ocs = r, ots = 1
// A cluster of kLoraSplit CTAs owns 32 columns; CTA s of the cluster runs
// over the s-th quarter of the rows in chunks of 64, through a ring of
// kLoraStages cp.async stages (the chunk of `in` as [i][c], read transposed
// with ldmatrix; the fp32 coefficients as [i][t], rounded to bf16 pairs when
// the B fragments are built).  Products accumulate in fp32 on mma.sync
// (M = columns, N = rank, K = rows), in row order; the cluster's partials are
// then added in rank order through distributed shared memory.
constexpr int kLoraSplit = 4;
constexpr int kLoraStages = 4;

template <int R8>
struct ColGradSmem {
    static constexpr int kMC = 64, kCT = 32;
    static constexpr int kInStride = kCT + 8;                  // bf16; 80-byte rows: conflict-free ldmatrix
    static constexpr int kCfStride = 8 * R8 + 4;               // fp32; 16-byte aligned, conflict-free pairs
    static constexpr int kInBytes = kMC * kInStride * 2;
    static constexpr int kCfBytes = kMC * kCfStride * 4;
    static constexpr int kStageBytes = kInBytes + kCfBytes;
    static constexpr int kBytes = kLoraStages * kStageBytes;
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}

template <int R8>
__global__ void __launch_bounds__(256) lora_colgrad_mma_kernel(const uint16_t* __restrict__ in, int64_t m,
                                                               int64_t ncols, const float* __restrict__ coef, int r,
                                                               float s, float* __restrict__ grad, int64_t ocs,
                                                               int64_t ots) {
    using L = ColGradSmem<R8>;
    constexpr int MC = L::kMC, CT = L::kCT, NP = 2 * R8;       // row chunk, columns, (m16, n8) tile pairs
    extern __shared__ __align__(128) uint8_t lora_smem[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, j = lane & 3;
    const int64_t c0 = static_cast<int64_t>(blockIdx.x) * CT;
    // this CTA's rows: a multiple of 64 per cluster rank
    const int64_t per = (m + static_cast<int64_t>(kLoraSplit) * MC - 1) / (static_cast<int64_t>(kLoraSplit) * MC) * MC;
    const int64_t rbeg = static_cast<int64_t>(blockIdx.y) * per;
    const int64_t rend = rbeg + per < m ? rbeg + per : m;
    const int nchunk = rend > rbeg ? static_cast<int>((rend - rbeg + MC - 1) / MC) : 0;
    const uint32_t sbase = static_cast<uint32_t>(__cvta_generic_to_shared(lora_smem));

    auto load_chunk = [&](int ci) {
        const int stage = ci % kLoraStages;
        const int64_t i0 = rbeg + static_cast<int64_t>(ci) * MC;
        const uint32_t sin = sbase + stage * L::kStageBytes, scf = sin + L::kInBytes;
        {   // 64 x 32 bf16 of `in`: one 16-byte piece per thread
            const int lr = threadIdx.x >> 2, lq = threadIdx.x & 3;
            const bool ok = i0 + lr < rend && c0 + 8 * lq < ncols;
            const uint16_t* src = ok ? in + (i0 + lr) * ncols + c0 + 8 * lq : in;
            cp_async16(sin + (lr * L::kInStride + 8 * lq) * 2, src, ok);
        }
        // 64 x r fp32 coefficients (r % 4 == 0 is not required: pieces past r read zeros)
        const int pieces = (8 * R8) / 4;
        for (int e = threadIdx.x; e < MC * pieces; e += blockDim.x) {
            const int lr = e / pieces, pq = e - lr * pieces;
            const bool ok = i0 + lr < rend && 4 * pq < r;
            const float* src = ok ? coef + (i0 + lr) * r + 4 * pq : coef;
            cp_async16(scf + (lr * L::kCfStride + 4 * pq) * 4, src, ok && (4 * pq + 4 <= r));
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };

    float acc[2][4];
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[u][e] = 0.0f;
#pragma unroll
    for (int ci = 0; ci < kLoraStages - 1; ++ci) {
        if (ci < nchunk) load_chunk(ci);
        else asm volatile("cp.async.commit_group;" ::: "memory");
    }
    for (int ci = 0; ci < nchunk; ++ci) {
        asm volatile("cp.async.wait_group %0;" ::"n"(kLoraStages - 2) : "memory");
        __syncthreads();                                       // chunk ci landed; chunk ci - 1 consumed
        if (ci + kLoraStages - 1 < nchunk) load_chunk(ci + kLoraStages - 1);
        else asm volatile("cp.async.commit_group;" ::: "memory");
        const int stage = ci % kLoraStages;
        const uint8_t* st_in = lora_smem + stage * L::kStageBytes;
        const float* st_cf = reinterpret_cast<const float*>(st_in + L::kInBytes);
        const uint32_t sin = sbase + stage * L::kStageBytes;
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int pidx = warp + 8 * u;
            if (pidx < NP) {
                const int mt = pidx & 1, nt = pidx >> 1;
                const int t = nt * 8 + g;
#pragma unroll
                for (int ks = 0; ks < MC / 16; ++ks) {
                    // A = in^T (rows c, columns i): four transposed 8x8 tiles
                    const int q = lane >> 3;
                    const uint32_t addr =
                        sin + ((ks * 16 + ((q >> 1) << 3) + (lane & 7)) * L::kInStride + mt * 16 + ((q & 1) << 3)) * 2;
                    uint32_t a0, a1, a2, a3;
                    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(a0), "=r"(a1), "=r"(a2), "=r"(a3)
                                 : "r"(addr));
                    // B = coef (rows i, columns t) rounded to bf16 pairs along i
                    const int i = ks * 16 + 2 * j;
                    const uint32_t b0 = pack_bf16x2_rn(st_cf[i * L::kCfStride + t], st_cf[(i + 1) * L::kCfStride + t]);
                    const uint32_t b1 =
                        pack_bf16x2_rn(st_cf[(i + 8) * L::kCfStride + t], st_cf[(i + 9) * L::kCfStride + t]);
                    lora_mma(acc[u], a0, a1, a2, a3, b0, b1);
                }
            }
        }
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();
    // cluster reduction in rank order: every CTA parks its tile in its own
    // shared memory, rank 0 adds them up and writes the result
    float* s_acc = reinterpret_cast<float*>(lora_smem);       // [32 columns][8 R8]
#pragma unroll
    for (int u = 0; u < 2; ++u) {
        const int pidx = warp + 8 * u;
        if (pidx < NP) {
            const int mt = pidx & 1, nt = pidx >> 1;
#pragma unroll
            for (int e = 0; e < 4; ++e)
                s_acc[(mt * 16 + g + 8 * (e >> 1)) * (8 * R8) + nt * 8 + 2 * j + (e & 1)] = acc[u][e];
        }
    }
    asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::: "memory");
    if (blockIdx.y == 0) {
        for (int e = threadIdx.x; e < CT * 8 * R8; e += blockDim.x) {
            const int cl = e / (8 * R8), t = e - cl * (8 * R8);
            float v = 0.0f;
            for (int rk = 0; rk < kLoraSplit; ++rk) {
                uint32_t remote;
                asm volatile("mapa.shared::cluster.u32 %0, %1, %2;"
                             : "=r"(remote)
                             : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(s_acc + e))), "r"(rk));
                float x;
                asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(x) : "r"(remote) : "memory");
                v += x;
            }
            const int64_t c = c0 + cl;
            if (c < ncols && t < r) grad[c * ocs + t * ots] = __fmul_rn(s, v);
        }
    }
    // keep every CTA's shared memory alive until rank 0 has read it
    asm volatile("barrier.cluster.arrive.release.aligned;\nbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

}  // namespace lbq
