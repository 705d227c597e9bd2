// quantize.cuh -- quantize/pack and dequantize kernels (HBM-bound, SIMT).
//
// MinMax group quantizer: GreenBit.AI low-bit LLM article, section 模型量化,
// step (1) (INT4 with group size 128, INT2 with group size 64).
// Packing (first code in the high bits): bitsandbytes FSDP-QLoRA guide,
// section 量化数据的存储.
// 4-bit codebook with per-64 absmax and double quantization of absmax:
// QLoRA explainer, sections 关键技术细节 and 结论; bitsandbytes guide (nf4,
// nested absmax).
//
// Every lane owns 8 consecutive elements (one 16-byte load of bf16), so a warp
// streams 512 contiguous bytes per step.  Group reductions (min/max, absmax)
// are warp shuffles over the lanes of one group.  Each fp32 step is written
// with an explicit round-to-nearest intrinsic so that the results are the
// IEEE single-precision results, bit for bit (the build also disables FMA
// contraction).
#pragma once

#include "common.cuh"

namespace lbq {

// rint(fl(w / d)), the IEEE quotient rounded half-to-even to an integer, for
// finite w and a positive normal d with rs = fl(1 / d).  t = fl(w * rs) is
// within 2 ulp of w / d and fl(w / d) within half an ulp, so rint(t) is the
// answer whenever t is more than 3 ulp away from the nearest half-integer.
// For |t| < 2^11 an ulp is at most 2^-13, so a fixed margin of 2^-10 covers
// the 3 ulp; only elements inside the margin (or with |t| >= 2^11) pay for
// the correctly rounded division.
__device__ __forceinline__ float rint_div(float w, float d, float rs) {
    const float t = __fmul_rn(w, rs);
    const float n = rintf(t);
    const float h = __fsub_rn(t, n);                                 // exact (Sterbenz): |h| <= 0.5
    if (fabsf(h) < 0.4990234375f && fabsf(t) < 2048.0f) return n;   // 0.5 - 2^-10
    return rintf(__fdiv_rn(w, d));
}

// ---------------------------------------------------------------------------
// MinMax quantize + pack.  Group = 128 (4 bit) or 64 (2 bit); one group is
// covered by GROUP/8 consecutive lanes.  The kernels issue about one
// instruction per cycle on most of their cycles (exact IEEE steps per
// element); the MinMax kernel also keeps the next two chunks' loads of a warp
// in flight while it processes the current one (a rolling prefetch, 3-6%
// faster; loading several chunks and then processing them all was slower).
// ---------------------------------------------------------------------------

// The grid-stride walk of a warp over 512-byte chunks (32 lanes x 16 bytes)
// with AHEAD chunks' loads in flight; fn(raw, chunk, valid) processes one
// lane's 16 bytes.
template <int AHEAD, typename F>
__device__ __forceinline__ void quant_chunk_loop(const uint4* __restrict__ W, int64_t nchunks, F&& fn) {
    const int lane = threadIdx.x & 31;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    int64_t base = static_cast<int64_t>(blockIdx.x) * blockDim.x + (threadIdx.x & ~31u);
    auto load = [&](int64_t b) {
        const int64_t chunk = b + lane;
        return chunk < nchunks ? __ldg(W + chunk) : make_uint4(0, 0, 0, 0);
    };
    uint4 buf[AHEAD + 1];
#pragma unroll
    for (int u = 0; u < AHEAD; ++u) buf[u] = load(base + u * stride);
    for (; base < nchunks; base += stride) {
        buf[AHEAD] = load(base + AHEAD * stride);
        fn(buf[0], base + lane, base + lane < nchunks);
#pragma unroll
        for (int u = 0; u < AHEAD; ++u) buf[u] = buf[u + 1];
    }
}

template <int BITS>
__device__ __forceinline__ void minmax_quantize_chunk(uint4 raw, int64_t chunk, bool valid, int lane,
                                                      uint8_t* __restrict__ packed, uint16_t* __restrict__ scale,
                                                      uint16_t* __restrict__ zero) {
    constexpr int GROUP = (BITS == 4) ? 128 : 64;
    constexpr int LPG = GROUP / 8;  // lanes per group
    constexpr float Q = static_cast<float>((1 << BITS) - 1);
    const uint32_t words[4] = {raw.x, raw.y, raw.z, raw.w};
    float v[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = bf16_bits_to_f32(words[i] & 0xFFFFu);
        v[2 * i + 1] = bf16_bits_to_f32(words[i] >> 16);
    }
    // the lane's extremes on bf16 pairs (exact: a minimum of bf16 values is one of them)
    __nv_bfloat162 mn2 = *reinterpret_cast<const __nv_bfloat162*>(&words[0]), mx2 = mn2;
#pragma unroll
    for (int i = 1; i < 4; ++i) {
        const __nv_bfloat162 x = *reinterpret_cast<const __nv_bfloat162*>(&words[i]);
        mn2 = __hmin2(mn2, x);
        mx2 = __hmax2(mx2, x);
    }
    float mn = fminf(__low2float(mn2), __high2float(mn2));
    float mx = fmaxf(__low2float(mx2), __high2float(mx2));
#pragma unroll
    for (int off = LPG / 2; off > 0; off >>= 1) {
        mn = fminf(mn, __shfl_xor_sync(0xFFFFFFFFu, mn, off));
        mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, off));
    }
    if (!valid) return;  // whole groups are either valid or not
    // -0 and +0 compare equal; adding +0 makes both extremes +0.
    mn = __fadd_rn(mn, 0.0f);
    mx = __fadd_rn(mx, 0.0f);
    const float r = __fsub_rn(mx, mn);
    uint16_t s16 = f32_to_f16_bits(__fdiv_rn(r, Q));
    if (r == 0.0f || (s16 & 0x7FFFu) == 0) s16 = 0x3C00u;  // 1.0
    const float sf = f16_bits_to_f32(s16);
    const uint16_t z16 = f32_to_f16_bits(rintf(__fdiv_rn(-mn, sf)));
    const float zf = f16_bits_to_f32(z16);
    uint32_t q[8];
    const float rs = __frcp_rn(sf);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float t = rint_div(v[i], sf, rs);
        t = __fadd_rn(t, zf);
        t = fminf(fmaxf(t, 0.0f), Q);
        q[i] = static_cast<uint32_t>(t);
    }
    if (BITS == 4) {
        uint32_t word = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) word |= ((q[2 * j] << 4) | q[2 * j + 1]) << (8 * j);
        reinterpret_cast<uint32_t*>(packed)[chunk] = word;
    } else {
        uint32_t half = 0;
#pragma unroll
        for (int j = 0; j < 2; ++j)
            half |= ((q[4 * j] << 6) | (q[4 * j + 1] << 4) | (q[4 * j + 2] << 2) | q[4 * j + 3]) << (8 * j);
        reinterpret_cast<uint16_t*>(packed)[chunk] = static_cast<uint16_t>(half);
    }
    if ((lane & (LPG - 1)) == 0) {
        const int64_t g = chunk / LPG;
        scale[g] = s16;
        zero[g] = z16;
    }
}

template <int BITS>
__global__ void __launch_bounds__(256) minmax_quantize_kernel(const uint4* __restrict__ W, int64_t nchunks,
                                                              uint8_t* __restrict__ packed,
                                                              uint16_t* __restrict__ scale,
                                                              uint16_t* __restrict__ zero) {
    const int lane = threadIdx.x & 31;
    quant_chunk_loop<2>(W, nchunks, [&](uint4 raw, int64_t chunk, bool valid) {
        minmax_quantize_chunk<BITS>(raw, chunk, valid, lane, packed, scale, zero);
    });
}

// ---------------------------------------------------------------------------
// Codebook quantize + pack.  Blocks of 64 consecutive elements (8 lanes).
// Also accumulates, per CTA, the fp64 sum of the block absmax values (used by
// double quantization; exact under the documented range condition).
// ---------------------------------------------------------------------------
// The table in code order c[0..15] (any order; equal entries allowed, such
// as the +0 and -0 of the FP4 table) as a search table: its distinct values
// in increasing order u[0..nu-1] (+inf after them), and for each the lowest
// code that holds it.  Returns false when the table breaks the preconditions:
// entries in [-1, 1], a zero among them, distinct values at least 2^-20
// apart (then the nearest-value search below equals the exhaustive
// search with its lower-index tie rule).  One thread builds it.
__device__ __forceinline__ bool codebook_search_table(const float* c, float* u, uint32_t* rep) {
    bool ok = true, has_zero = false;
    int nu = 0;
    for (int j = 0; j < 16; ++j) {
        has_zero |= (c[j] == 0.0f);
        ok &= (c[j] >= -1.0f) && (c[j] <= 1.0f);
        // insert value c[j] (code j) unless an equal value is already there
        // (codes are visited in increasing order, so the first code stays)
        int pos = 0;
        while (pos < nu && u[pos] < c[j]) ++pos;
        if (pos < nu && u[pos] == c[j]) continue;
        for (int i = nu; i > pos; --i) {
            u[i] = u[i - 1];
            rep[i] = rep[i - 1];
        }
        u[pos] = c[j];
        rep[pos] = static_cast<uint32_t>(j);
        ++nu;
    }
    for (int i = 1; i < nu; ++i) ok &= (u[i] - u[i - 1]) >= 9.5367431640625e-07f;
    for (int i = nu; i < 16; ++i) {
        u[i] = __int_as_float(0x7f800000);   // +inf: never below x, never nearest
        rep[i] = 15u;
    }
    return ok && has_zero;
}

// Code of the entry nearest to x, the lower code on a tie.  The search
// table is sorted, so the nearest value is one of the two that bracket x.
__device__ __forceinline__ uint32_t nearest_code(const float* u, const uint32_t* rep, float x) {
    int j = -1;
    if (u[j + 8] <= x) j += 8;
    if (u[j + 4] <= x) j += 4;
    if (u[j + 2] <= x) j += 2;
    if (u[j + 1] <= x) j += 1;
    if (j < 0) return rep[0];
    if (j == 15) return rep[15];
    const float d0 = fabsf(__fsub_rn(x, u[j]));
    const float d1 = fabsf(__fsub_rn(x, u[j + 1]));
    if (d1 < d0) return rep[j + 1];
    if (d0 < d1) return rep[j];
    return min(rep[j], rep[j + 1]);
}

__global__ void __launch_bounds__(256) codebook_quantize_kernel(const uint4* __restrict__ W, int64_t nchunks,
                                                                const float* __restrict__ codebook,
                                                                uint8_t* __restrict__ packed,
                                                                float* __restrict__ absmax,
                                                                double* __restrict__ cta_sums) {
    __shared__ float s_cb[16];
    __shared__ float s_u[16];
    __shared__ uint32_t s_rep[16];
    __shared__ double s_sum[8];
    if (threadIdx.x < 16) s_cb[threadIdx.x] = codebook[threadIdx.x];
    __syncthreads();
    if (threadIdx.x == 0) {
        const bool ok = codebook_search_table(s_cb, s_u, s_rep);
        if (blockIdx.x == 0 && !ok) record_status(kStatusBadTable);
    }
    __syncthreads();
    const int lane = threadIdx.x & 31;
    double my_sum = 0.0;
    auto process = [&](uint4 raw, int64_t chunk, bool valid) {
        const uint32_t words[4] = {raw.x, raw.y, raw.z, raw.w};
        float v[8];
        float a = 0.0f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[2 * i] = bf16_bits_to_f32(words[i] & 0xFFFFu);
            v[2 * i + 1] = bf16_bits_to_f32(words[i] >> 16);
            a = fmaxf(a, fmaxf(fabsf(v[2 * i]), fabsf(v[2 * i + 1])));
        }
#pragma unroll
        for (int off = 4; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, off));
        if (!valid) return;
        uint32_t word = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float x0 = (a == 0.0f) ? 0.0f : __fdiv_rn(v[2 * j], a);
            const float x1 = (a == 0.0f) ? 0.0f : __fdiv_rn(v[2 * j + 1], a);
            word |= ((nearest_code(s_u, s_rep, x0) << 4) | nearest_code(s_u, s_rep, x1)) << (8 * j);
        }
        reinterpret_cast<uint32_t*>(packed)[chunk] = word;
        if ((lane & 7) == 0) {
            absmax[chunk >> 3] = a;
            my_sum += static_cast<double>(a);
        }
    };
    quant_chunk_loop<0>(W, nchunks, process);
    if (cta_sums != nullptr) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) my_sum += __shfl_xor_sync(0xFFFFFFFFu, my_sum, off);
        if (lane == 0) s_sum[threadIdx.x >> 5] = my_sum;
        __syncthreads();
        if (threadIdx.x == 0) {
            double t = 0.0;
            for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) t += s_sum[w];
            cta_sums[blockIdx.x] = t;
        }
    }
}

// offset = fp32(fp64 sum / nb): one CTA sums the per-CTA partial sums.
__global__ void __launch_bounds__(256) absmax_offset_kernel(const double* __restrict__ cta_sums, int nparts,
                                                            int64_t nb, float* __restrict__ offset) {
    __shared__ double s[256];
    double t = 0.0;
    for (int i = threadIdx.x; i < nparts; i += blockDim.x) t += cta_sums[i];
    s[threadIdx.x] = t;
    __syncthreads();
    for (int w = blockDim.x / 2; w > 0; w >>= 1) {
        if (threadIdx.x < w) s[threadIdx.x] += s[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) *offset = __double2float_rn(__ddiv_rn(s[0], static_cast<double>(nb)));
}

// Double quantization: per block of 256 absmax values, s2 = max |a - offset|
// and q8 = clamp(rint(((a - offset) / s2) * 127), -127, 127).
__global__ void __launch_bounds__(256) double_quant_kernel(const float* __restrict__ absmax, int64_t nb,
                                                           const float* __restrict__ offset,
                                                           int8_t* __restrict__ q8, float* __restrict__ s2) {
    __shared__ float s_max[8];
    const int64_t i = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
    const float off = *offset;
    const float c = (i < nb) ? __fsub_rn(absmax[i], off) : 0.0f;
    float m = fabsf(c);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if ((threadIdx.x & 31) == 0) s_max[threadIdx.x >> 5] = m;
    __syncthreads();
    m = s_max[0];
#pragma unroll
    for (int w = 1; w < 8; ++w) m = fmaxf(m, s_max[w]);
    if (i < nb) {
        float qf = 0.0f;
        if (m != 0.0f) {
            qf = rintf(__fmul_rn(__fdiv_rn(c, m), 127.0f));
            qf = fminf(fmaxf(qf, -127.0f), 127.0f);
        }
        q8[i] = static_cast<int8_t>(qf);
    }
    if (threadIdx.x == 0) s2[blockIdx.x] = m;
}

// ---------------------------------------------------------------------------
// Dequantize to fp32 (the parity target of the fused kernels).
// ---------------------------------------------------------------------------
template <int BITS>
__global__ void __launch_bounds__(256) minmax_dequantize_kernel(const uint8_t* __restrict__ packed,
                                                                const uint16_t* __restrict__ scale,
                                                                const uint16_t* __restrict__ zero,
                                                                int64_t nchunks, float4* __restrict__ out) {
    constexpr int LPG = ((BITS == 4) ? 128 : 64) / 8;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; c < nchunks; c += stride) {
        uint32_t q[8];
        if (BITS == 4) {
            const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(packed) + c);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                q[2 * j] = (w >> (8 * j + 4)) & 15u;
                q[2 * j + 1] = (w >> (8 * j)) & 15u;
            }
        } else {
            const uint32_t w = __ldg(reinterpret_cast<const uint16_t*>(packed) + c);
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int t = 0; t < 4; ++t) q[4 * j + t] = (w >> (8 * j + 6 - 2 * t)) & 3u;
        }
        const int64_t g = c / LPG;
        const float sf = f16_bits_to_f32(__ldg(scale + g));
        const float zf = f16_bits_to_f32(__ldg(zero + g));
        float r[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) r[i] = __fmul_rn(__fsub_rn(static_cast<float>(q[i]), zf), sf);
        out[2 * c] = make_float4(r[0], r[1], r[2], r[3]);
        out[2 * c + 1] = make_float4(r[4], r[5], r[6], r[7]);
    }
}

// absmax' = ((q8 / 127) * s2) + offset, three fp32 operations.
__device__ __forceinline__ float double_dequant(int8_t q8, float s2, float off) {
    return __fadd_rn(__fmul_rn(__fdiv_rn(static_cast<float>(q8), 127.0f), s2), off);
}

__global__ void __launch_bounds__(256) codebook_dequantize_kernel(const uint8_t* __restrict__ packed,
                                                                  const float* __restrict__ absmax,
                                                                  const int8_t* __restrict__ q8,
                                                                  const float* __restrict__ s2,
                                                                  const float* __restrict__ offset,
                                                                  const float* __restrict__ codebook,
                                                                  int64_t nchunks, float4* __restrict__ out) {
    __shared__ float s_cb[16];
    if (threadIdx.x < 16) s_cb[threadIdx.x] = codebook[threadIdx.x];
    __syncthreads();
    const float off = (q8 != nullptr) ? *offset : 0.0f;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t c = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; c < nchunks; c += stride) {
        const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(packed) + c);
        const int64_t b = c >> 3;  // block of 64 elements
        const float a = (q8 != nullptr) ? double_dequant(q8[b], s2[b >> 8], off) : __ldg(absmax + b);
        float r[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            r[2 * j] = __fmul_rn(s_cb[(w >> (8 * j + 4)) & 15u], a);
            r[2 * j + 1] = __fmul_rn(s_cb[(w >> (8 * j)) & 15u], a);
        }
        out[2 * c] = make_float4(r[0], r[1], r[2], r[3]);
        out[2 * c + 1] = make_float4(r[4], r[5], r[6], r[7]);
    }
}

}  // namespace lbq
